/*
 * ssd.h -- C ABI of libssd.so, a B200 (sm_100a) implementation of the
 * Mamba-2 / SSD selective-state-space mixer scan.
 *
 * The operation (per batch row b and head h, tokens t = 0 .. L-1):
 *
 *   u        = SiLU(causal depthwise conv, kernel 4, over the x|B|C channels)
 *              -- "Mini-K3-1H-mamba2-n64-g8" model card, Architecture; the
 *              channel order x|B|C and conv_dim = H*P + 2*G*N follow the
 *              codestral_mamba.ts weight-port header.  With dconv = 1 there
 *              is no conv and no SiLU (mojolearn Mamba3Block: "v is the raw
 *              x split").
 *   B_t, C_t = optional RMSNorm (eps 1e-5) * weight + per-head bias
 *              (mojolearn Mamba3Block, class description and Parameters)
 *   dt_t     = softplus(dt_raw_t + dt_bias[h]), no clamp (falcon_mamba.ts
 *              header; Mamba3Block "no dt clamp")
 *   a_t      = A[h], or per token max-magnitude-floored: min(A[b,t,h], -1e-4)
 *              (Mamba3Block "A floor 1e-4")
 *   h_t      = exp(dt_t a_t) h_{t-1} + dt_t x_t (outer) B_t      (P x N, fp32)
 *   y_t      = C_t . h_t + D[h] x_t ;   out_t = y_t * SiLU(z_t)
 *
 * and the state restarts from zero (and the conv sees no earlier token) at
 * every packed-document boundary: a position whose seq_idx differs from its
 * left neighbour's (model card, "Checkpoint and training").  The caller's
 * initial state belongs to the first document of each row.
 *
 * Conventions for every call:
 *  - All tensor pointers are DEVICE pointers owned by the caller, contiguous
 *    and row-major as described per argument.  Activation tensors (x, z, B,
 *    C, out, conv_w, conv_b and the conv part of a state buffer) have the
 *    handle's act_dtype; dt_raw, dt_bias, A, D, norm weights and the SSM
 *    state are fp32; seq_idx is int32.
 *  - x, z, B, C, out and state buffers must be 16-byte aligned; the other
 *    pointers 4-byte aligned.
 *  - Work is enqueued asynchronously on `stream` (a cudaStream_t; NULL is the
 *    legacy default stream).  A handle serves one stream at a time.
 *  - Calls may be captured into a CUDA graph (stream capture).  A graph
 *    replays every call with the argument values and the handle workspace of
 *    its capture, so replays of a graph must not overlap on the GPU with
 *    each other or with other calls on the same handle.  A captured fused
 *    forward clears its segment hand-off flags inside the graph, so every
 *    replay waits for its own hand-offs.
 *  - Arguments are validated on the host before anything is launched: a call
 *    that returns an error status launched nothing and touched no memory.
 *    ssd_last_error() then names the offending argument (the calling thread's
 *    message).  Errors raised on the device by an accepted call are reported
 *    by ssd_check().
 *  - Calls allocate nothing: ssd_create sizes the handle's workspace for
 *    max_batch x max_seqlen.
 */
#ifndef SSD_H
#define SSD_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

struct CUstream_st;                 /* cudaStream_t is struct CUstream_st* */
typedef struct ssd_handle ssd_handle;

typedef enum {
    SSD_OK = 0,
    SSD_ERR_INVALID_ARG = 1,        /* null/ill-formed argument, bad shape */
    SSD_ERR_UNSUPPORTED = 2,        /* well-formed but not implemented (e.g. headdim % 8) */
    SSD_ERR_ALIGNMENT = 3,          /* pointer not aligned as required */
    SSD_ERR_SHAPE_EXCEEDS_MAX = 4,  /* batch/seqlen above the handle's maxima */
    SSD_ERR_CUDA = 5,               /* a CUDA runtime call failed */
    SSD_ERR_DEVICE = 6              /* ssd_check: the device reported an error */
} ssd_status;

typedef enum { SSD_DTYPE_F32 = 0, SSD_DTYPE_BF16 = 1 } ssd_dtype;
typedef enum { SSD_A_PER_HEAD = 0, SSD_A_PER_TOKEN = 1 } ssd_a_mode;

/* Which kernel sequence ssd_forward runs.
 *  FUSED : one persistent chunk-sweep kernel per (row, head) that keeps the
 *          running state on chip (tcgen05 tensor-core contractions, bf16
 *          operands, fp32 accumulation); bf16 activations, headdim 64,
 *          d_state 64 or 128.  With bc_norm, each head's normalised B and C
 *          tiles are built in shared memory and never written to memory.
 *  STAGED: the five-stage pipeline conv -> dt/cumsum -> chunk states ->
 *          state passing -> chunk outputs, fp32 accumulation throughout (the
 *          chunk-state and chunk-output contractions on the tensor cores with
 *          tf32 operands for bf16 activations, as fp32 products for fp32
 *          activations); any supported shape and both dtypes.  It writes
 *          every chunk state to memory and reads it back, so it is several
 *          times slower than FUSED on the shapes both serve (about 4.7x on a
 *          32-head, d_state 64 layer; 6x at d_state 128): read ssd_get_path
 *          after ssd_create when throughput matters.
 *  AUTO  : FUSED when the shape and dtype allow it, else STAGED. */
typedef enum { SSD_PATH_AUTO = 0, SSD_PATH_FUSED = 1, SSD_PATH_STAGED = 2 } ssd_path;

typedef struct {
    int32_t nheads;      /* H >= 1 */
    int32_t headdim;     /* P, multiple of 8, <= 128 */
    int32_t dstate;      /* N, multiple of 8, <= 256 */
    int32_t ngroups;     /* G, divides H; head h uses B/C group h / (H / G) */
    int32_t dconv;       /* 1 (no conv) or 4 */
    int32_t chunk;       /* 0 or 64 (the chunk length of the chunked scan) */
    int32_t act_dtype;   /* ssd_dtype */
    int32_t a_mode;      /* ssd_a_mode */
    int32_t bc_norm;     /* 1: B/C RMSNorm + per-head bias, see ssd_set_bc_norm */
    int32_t max_batch;   /* >= 1 */
    int32_t max_seqlen;  /* >= 1 */
    int32_t path;        /* ssd_path */
    int32_t validate_finite;  /* 1: after every forward / step, scan out and the
                                 fp32 state for NaN or infinity; ssd_check then
                                 reports SSD_ERR_DEVICE.  Costs one extra read of
                                 the results.  0: no check. */
} ssd_desc;

/* Create a handle for one layer shape.  Validates d, picks the path, and
 * allocates (cudaMalloc, on the current device) the workspace every later
 * call uses.  On success *out owns that memory until ssd_destroy. */
ssd_status ssd_create(const ssd_desc* d, ssd_handle** out);

/* Free the handle's workspace and the handle; NULL is a no-op.  The caller
 * must make sure no call on the handle is still running on the GPU. */
void ssd_destroy(ssd_handle* h);

/* The path ssd_create chose (SSD_PATH_FUSED or SSD_PATH_STAGED), or -1. */
int32_t ssd_get_path(const ssd_handle* h);

/* B/C normalisation parameters (Mamba3Block Parameters: B_norm.weight,
 * C_norm.weight (N); B_bias, C_bias (H, N)), device fp32 pointers that must
 * stay valid while calls run.  NULL weight = ones, NULL bias = zeros.  Only
 * for handles created with bc_norm = 1. */
ssd_status ssd_set_bc_norm(ssd_handle* h, const float* B_norm_w, const float* C_norm_w,
                           const float* B_bias, const float* C_bias);

/* Gated RMSNorm after the scan (the upstream Mamba-2 block's norm(y * silu(z));
 * codestral_mamba.ts header: `mixer.norm.weight [d_inner]`, reconciliation 3).
 * With enable = 1, every later ssd_forward / ssd_forward_ragged / ssd_step
 * rewrites out in place as out * weight / sqrt(mean(out^2) + eps), the mean
 * taken over each group of group_size consecutive channels of a token
 * (group_size 0 = H*P, one norm per token; otherwise it must divide H*P, be a
 * multiple of 8 and be at most 16384).  weight: (H*P) fp32 device pointer,
 * 16-byte aligned, that stays valid while calls run, or NULL (ones).  eps in [0, 1]; the Mamba3Block
 * norms use 1e-5.  Padding tokens of a ragged batch stay +0.0.  enable = 0
 * turns the norm off (the other arguments are then ignored).  The norm adds one
 * read and one write of out; validate_finite checks the normed out. */
ssd_status ssd_set_gated_norm(ssd_handle* h, int32_t enable, const float* weight,
                              int32_t group_size, float eps);

/* Bytes of one state buffer for `batch` rows: the fp32 SSM state
 * (batch, H, P, N), then, at ssd_state_conv_offset, the conv history
 * (batch, dconv-1, conv_dim) in act_dtype, oldest token first (absent when
 * dconv = 1).  An all-zero buffer is a fresh state (Mamba3Block.allocate_state). */
size_t ssd_state_bytes(const ssd_handle* h, int32_t batch);
size_t ssd_state_conv_offset(const ssd_handle* h, int32_t batch);

/*
 * Forward over `seqlen` tokens of `batch` rows (Mamba3Block.forward with a
 * state: read at entry, written at exit).
 *   x, z, out   (batch, seqlen, H*P)   channel h*P + p
 *   dt_raw      (batch, seqlen, H)     fp32
 *   dt_bias, D  (H)                    fp32
 *   A           (H) fp32, already negative (A = -exp(A_log), codestral_mamba.ts
 *               reconciliation 2), or (batch, seqlen, H) when a_mode = PER_TOKEN
 *   B, C        (batch, seqlen, G*N)
 *   conv_w      (conv_dim, dconv), conv_b (conv_dim), x|B|C channel order; w[c, dconv-1]
 *               multiplies the current token.  NULL iff dconv = 1.
 *   seq_idx     (batch, seqlen) int32 document ids, or NULL (one document per row)
 *   init_state  state buffer (ssd_state_bytes) read at entry, or NULL (zeros)
 *   final_state state buffer written at exit, or NULL; may equal init_state
 *   out         may not alias any input
 * Returns SSD_OK or an error before any launch (see above).
 */
ssd_status ssd_forward(ssd_handle* h, int32_t batch, int32_t seqlen,
                       const void* x, const void* z, const float* dt_raw, const float* dt_bias,
                       const float* A, const void* B, const void* C, const float* D,
                       const void* conv_w, const void* conv_b, const int32_t* seq_idx,
                       const void* init_state, void* out, void* final_state,
                       struct CUstream_st* stream);

/*
 * Forward over a ragged batch: row b holds lengths[b] real tokens (a device
 * int32 array of `batch` entries, each clamped to [0, seqlen]); the rest of
 * the row is padding that is not part of the sequence.  Padding outputs are
 * written as +0.0, and the final state and conv history are those after the
 * row's last real token (a zero-length row hands init_state through).  Every
 * other argument is as for ssd_forward; lengths may not be NULL.
 */
ssd_status ssd_forward_ragged(ssd_handle* h, int32_t batch, int32_t seqlen, const int32_t* lengths,
                              const void* x, const void* z, const float* dt_raw,
                              const float* dt_bias, const float* A, const void* B, const void* C,
                              const float* D, const void* conv_w, const void* conv_b,
                              const int32_t* seq_idx, const void* init_state, void* out,
                              void* final_state, struct CUstream_st* stream);

/*
 * Forward over a packed in_proj output, read in place through row strides
 * (codestral_mamba.ts header: the Mamba-2 in_proj row splits as
 * [gate z | x|B|C | dt]).  zxbcdt is (batch, seqlen, ld) in act_dtype, and each
 * token's row holds, from column 0: z (H*P), x (H*P), B (G*N), C (G*N) and
 * dt_raw (H, in act_dtype rather than fp32); columns from 2*H*P + 2*G*N + H up
 * to ld are ignored.  ld * element size must be a multiple of 16 bytes and
 * zxbcdt 16-byte aligned.  Everything else is as for ssd_forward: the results
 * equal ssd_forward over the same values split into contiguous tensors.
 */
ssd_status ssd_forward_packed(ssd_handle* h, int32_t batch, int32_t seqlen, const void* zxbcdt,
                              int64_t ld, const float* dt_bias, const float* A, const float* D,
                              const void* conv_w, const void* conv_b, const int32_t* seq_idx,
                              const void* init_state, void* out, void* final_state,
                              struct CUstream_st* stream);

/*
 * One decode token per row (Mamba3Block.step: the same computation as forward
 * at L = 1 with the state carried).  Inputs are the forward's with seqlen 1:
 * x, z, out (batch, H*P); B, C (batch, G*N); dt_raw (batch, H); A (H) or
 * (batch, H).  `state` is required and updated in place.
 */
ssd_status ssd_step(ssd_handle* h, int32_t batch,
                    const void* x, const void* z, const float* dt_raw, const float* dt_bias,
                    const float* A, const void* B, const void* C, const float* D,
                    const void* conv_w, const void* conv_b, void* state, void* out,
                    struct CUstream_st* stream);

/*
 * Stage entry points: run one stage of the staged path alone, for stage-level
 * checks and profiling.
 *   ssd_stage_conv : u (batch, seqlen, conv_dim) fp32 = SiLU(conv) of x|B|C
 *                    (the first stage; init_state as in ssd_forward).
 *   ssd_stage_dt   : dt (batch, H, seqlen) fp32 = softplus(dt_raw + dt_bias) and
 *                    acs (batch, H, seqlen) fp32 = cumulative sum of dt*a restarted
 *                    at every chunk start (64 tokens) and at every document
 *                    boundary of seq_idx (NULL = none).
 */
ssd_status ssd_stage_conv(ssd_handle* h, int32_t batch, int32_t seqlen, const void* x,
                          const void* B, const void* C, const void* conv_w, const void* conv_b,
                          const int32_t* seq_idx, const void* init_state, float* u,
                          struct CUstream_st* stream);
ssd_status ssd_stage_dt(ssd_handle* h, int32_t batch, int32_t seqlen, const float* dt_raw,
                        const float* dt_bias, const float* A, const int32_t* seq_idx, float* dt,
                        float* acs, struct CUstream_st* stream);

/* Measurement hook.  When start and stop are cudaEvent_t handles (created by
 * the caller), every later ssd_forward / ssd_step records `start` on its
 * stream just before its main kernel (the fused chunk sweep, the staged
 * chunk-output kernel, or the decode kernel) and `stop` just after it, so
 * cudaEventElapsedTime gives that kernel's device time.  NULL, NULL turns the
 * hook off.  The events stay owned by the caller. */
ssd_status ssd_set_timing_events(ssd_handle* h, void* start, void* stop);

/* Testing hook for the failure path of the FUSED kernel, whose CTAs hand each
 * segment's leaving state to the next segment through a flag in device memory
 * and wait for it with a bounded spin.  wait_limit_ns sets the bound of every
 * wait of that kernel (0: the default of 1 s; otherwise at least 100000 ns),
 * and withhold_stream >= 0 makes the kernel never publish the first hand-off
 * of that (row * H + head) stream, so the wait for it runs out: the kernel then
 * raises the timeout bit of the device status word, lets its own copies and
 * tensor-core work finish, and exits; ssd_check reports SSD_ERR_DEVICE and the
 * outputs of that call are invalid.  -1 publishes every hand-off.  For
 * ssd_step the same two settings apply to the decode kernel, whose blocks wait
 * for bulk copies of their state: withhold_stream >= 0 makes the block of
 * (row * G + group) never request its first state piece, so its wait runs out;
 * that step's outputs, and that block's state and conv history, are then
 * invalid.  Nothing faults or hangs, and the next call on the handle is
 * unaffected. */
ssd_status ssd_set_wait_test(ssd_handle* h, uint64_t wait_limit_ns, int32_t withhold_stream);

/* Number of kernels this handle has launched since ssd_create. */
uint64_t ssd_launch_count(const ssd_handle* h);

/* Wait for `stream`, then read and clear the handle's device status word.
 * SSD_ERR_DEVICE when a kernel reported an error -- a bounded wait that timed
 * out, a rejected launch shape, or (validate_finite) a NaN or infinity in the
 * results; ssd_last_error says which -- and SSD_ERR_CUDA when the stream
 * itself failed. */
ssd_status ssd_check(ssd_handle* h, struct CUstream_st* stream);

/*
 * Gradients of the backward, all fp32 device buffers owned by the caller, each
 * with the layout of the input it belongs to.  x, z, B, C and dt_raw are
 * required; a NULL weight gradient is not computed.
 */
typedef struct {
    float* x;         /* (batch, seqlen, H*P) */
    float* z;         /* (batch, seqlen, H*P) */
    float* B;         /* (batch, seqlen, G*N) */
    float* C;         /* (batch, seqlen, G*N) */
    float* dt_raw;    /* (batch, seqlen, H) */
    float* dt_bias;   /* (H) */
    float* A;         /* (H), or (batch, seqlen, H) when a_mode = PER_TOKEN */
    float* D;         /* (H) */
    float* conv_w;    /* (conv_dim, 4); NULL when dconv = 1 */
    float* conv_b;    /* (conv_dim); NULL when dconv = 1 */
    float* B_norm_w;  /* (N); only with bc_norm */
    float* C_norm_w;  /* (N); only with bc_norm */
    float* B_bias;    /* (H, N); only with bc_norm */
    float* C_bias;    /* (H, N); only with bc_norm */
} ssd_grads;

/* Bytes of the device workspace ssd_backward needs for `batch` rows of
 * `seqlen` tokens (0 for a NULL handle or negative sizes). */
size_t ssd_backward_workspace_bytes(const ssd_handle* h, int32_t batch, int32_t seqlen);

/*
 * Backward of a zero-state prefill (mojolearn Mamba3Block, method "backward":
 * the gradients of the loss with respect to the input and every weight, given
 * the gradient of the output): the vector-Jacobian product of ssd_forward with
 * no initial state, without a final-state cotangent.  The model card's gate
 * ("Checkpoint and training") holds: a loss on one packed document gives
 * exactly zero gradient on every other document's inputs.
 *   x .. seq_idx  as for ssd_forward (lengths: as for ssd_forward_ragged, or
 *                 NULL; padding tokens take no gradient and their gout is ignored)
 *   gout          (batch, seqlen, H*P) act_dtype: gradient of the loss w.r.t. out
 *   grads         the outputs (see ssd_grads); written, not accumulated
 *   workspace     device memory of at least ssd_backward_workspace_bytes(h, batch,
 *                 seqlen) bytes, 256-byte aligned, owned by the caller; its
 *                 contents on entry do not matter
 * With bc_norm, the handle's ssd_set_bc_norm parameters are used and their
 * gradients can be asked for.  The arithmetic is fp32 throughout: the forward
 * quantities are recomputed by the staged kernels, and weight gradients are
 * summed in a fixed order, so a call repeats bit for bit.  headdim <= 64 and
 * dstate <= 128 (else SSD_ERR_UNSUPPORTED).  Asynchronous on `stream`; the
 * timing hook (ssd_set_timing_events) brackets the backward kernels that follow
 * the forward recompute.
 */
ssd_status ssd_backward(ssd_handle* h, int32_t batch, int32_t seqlen, const int32_t* lengths,
                        const void* x, const void* z, const float* dt_raw, const float* dt_bias,
                        const float* A, const void* B, const void* C, const float* D,
                        const void* conv_w, const void* conv_b, const int32_t* seq_idx,
                        const void* gout, const ssd_grads* grads, void* workspace,
                        size_t workspace_bytes, struct CUstream_st* stream);

/*
 * Allocation-free forward.  The method's pages have no counterpart to this
 * entry point: it computes what ssd_forward computes on the FUSED path (same
 * kernels, same arguments, same results), for callers that cannot allocate
 * device memory and so cannot create a handle -- code that runs under a
 * device-memory budget owned by someone else (a server that pre-sizes one
 * pool for its whole life and refuses later cudaMalloc calls), and code on a
 * latency-bound loop that cannot afford the device-wide synchronisation a
 * cudaFree implies.
 *
 * Scratch: a static device array of 64 MiB per device that belongs to the
 * loaded library (no cudaMalloc, cudaFree or allocating library call is
 * made).  Because the array is part of the library's device code, every
 * device on which that code is loaded holds the 64 MiB until the process
 * exits, whether or not this entry point is ever called: from the library's
 * first kernel launch on the device under lazy module loading (the CUDA
 * default), from its load under eager loading.  It holds 4 KiB of hand-off flags, then the segment hand-off states
 * (64 * dstate fp32 per slot; at least one slot per (row, head) stream, at
 * most 1024 slots), dt and the chunk cumsum ((batch, H, seqlen) fp32 each)
 * and, when dconv = 4, the convolved B|C ((batch, seqlen, 2*G*N) bf16).
 * A shape with more than 1024 streams (batch * H) or whose buffers exceed
 * the 64 MiB returns SSD_ERR_SHAPE_EXCEEDS_MAX before any launch; for H = 32,
 * G = 8, N = 64 that is about 28,000 tokens (batch * seqlen).
 *
 *   d           as for ssd_create; the shape must suit the FUSED path (bf16
 *               activations, headdim 64, dstate 64 or 128, bc_norm 0; path
 *               AUTO or FUSED, else SSD_ERR_UNSUPPORTED), and batch / seqlen
 *               must respect max_batch / max_seqlen as with a handle.
 *   x .. final_state, stream: as for ssd_forward.
 *   status      device pointer to one int32 that the caller owns (required);
 *               the kernels OR into it the bits ssd_check reports (1: a bounded
 *               wait timed out and the outputs are invalid; 2: a kernel rejected
 *               its launch shape; 4: with validate_finite, a NaN or infinity in
 *               out or the final state).  This call neither reads nor clears it.
 *
 * The first call on each device does a one-time set-up with that device
 * current: it looks up the array's device address (cudaGetSymbolAddress) and
 * clears the flag words on `stream`.  Make that first call before any stream
 * capture.  Every call on a device uses the same array, so calls that
 * overlap on the GPU (on different streams without an ordering between
 * them) race; calls on one stream, or ordered by events, do not.
 */
ssd_status ssd_forward_noalloc(const ssd_desc* d, int32_t batch, int32_t seqlen,
                               const void* x, const void* z, const float* dt_raw,
                               const float* dt_bias, const float* A, const void* B, const void* C,
                               const float* D, const void* conv_w, const void* conv_b,
                               const int32_t* seq_idx, const void* init_state, void* out,
                               void* final_state, int32_t* status, struct CUstream_st* stream);

/*
 * Mamba-1 selective scan (S6), the scan of the Falcon-Mamba port (falcon_mamba.ts
 * header: a Mamba-1 / S6 model; A = -exp(clamp(A_log, -10, 5)) as
 * selective_scan.ts computes it; dt = softplus(dt + bias)).  Per row b and
 * channel d (d_inner channels, state size dstate):
 *   h[n] <- exp(dt A[d,n]) h[n] + dt u B[n];  y = C.h + D[d] u;  out = y SiLU(z)
 * No handle: the call allocates nothing and keeps no state between calls.
 *   u, z, out   (batch, seqlen, d_inner) act_dtype; u is the convolved input,
 *               z NULL = no gate; out may not alias an input
 *   delta       (batch, seqlen, d_inner) fp32, before softplus
 *   delta_bias, D (d_inner) fp32;  A_log (d_inner, dstate) fp32
 *   B, C        (batch, seqlen, dstate) act_dtype, shared by every channel
 *   init_state, final_state  (batch, d_inner, dstate) fp32, or NULL (zeros / not
 *               written); they may be the same buffer
 *   dstate      8, 16 or 32 (else SSD_ERR_UNSUPPORTED); act_dtype an ssd_dtype
 * All pointers are contiguous row-major device memory that the caller owns,
 * aligned to their element size; the call is asynchronous on `stream`.
 * batch = 0 is a no-op; seqlen = 0 copies init_state to final_state (zeros
 * without an initial state).  Arguments are validated before any launch, as
 * for ssd_forward, and a refusal names the argument (ssd_last_error).
 */
ssd_status ssd_s6_forward(int32_t batch, int32_t seqlen, int32_t d_inner, int32_t dstate,
                          int32_t act_dtype, const void* u, const float* delta,
                          const float* delta_bias, const float* A_log, const void* B,
                          const void* C, const float* D, const void* z, const float* init_state,
                          void* out, float* final_state, struct CUstream_st* stream);

/* Measurement aid: the device's throughput of the hardware base-2 exponential
 * (the MUFU pipe), in results per second, from one timed kernel of independent
 * ex2 chains on `stream` (the call waits for it).  The Mamba-1 scan takes one
 * exponential per state and token, so this rate is its compute roofline. */
ssd_status ssd_ex2_throughput(double* results_per_second, struct CUstream_st* stream);

/* The calling thread's last error message ("" when none). */
const char* ssd_last_error(void);

/* A static name for a status code. */
const char* ssd_status_string(ssd_status s);

#ifdef __cplusplus
}
#endif
#endif /* SSD_H */
