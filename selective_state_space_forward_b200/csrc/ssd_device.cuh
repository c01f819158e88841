// ssd_device.cuh -- device helpers shared by the libssd kernels (sm_100a).
#pragma once
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace ssd {

typedef __nv_bfloat16 bf16;

constexpr int kChunk = 64;        // chunk length of the chunked scan
constexpr int kConvK = 4;         // causal conv kernel width when the conv is on
constexpr float kAFloor = 1e-4f;  // per-token |A| floor (Mamba3Block "A floor 1e-4")
constexpr float kNormEps = 1e-5f; // B/C RMSNorm epsilon (Mamba3Block Parameters)
constexpr float kChunkReset = -1.0f;  // carry factor of a chunk holding a document boundary

__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(bf16 v) { return __bfloat162float(v); }
template <typename T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ bf16 from_f<bf16>(float v) { return __float2bfloat16_rn(v); }

// x * sigmoid(x), with an IEEE divide so fp32 stages stay near correctly rounded.
__device__ __forceinline__ float silu_f(float v) { return v / (1.0f + expf(-v)); }

// SiLU(v) = v (1 + tanh(v/2)) / 2 = h + h tanh(h) with h = v/2, one hardware
// tanh (PTX tanh.approx, relative error ~2^-11): for results that are rounded
// to bf16 anyway.
__device__ __forceinline__ float silu_t(float v)
{
    const float h = 0.5f * v;
    float t;
    asm("tanh.approx.f32 %0, %1;" : "=f"(t) : "f"(h));
    return fmaf(h, t, h);
}

// 2^x, hardware approximation (PTX ex2.approx).
__device__ __forceinline__ float ex2(float x)
{
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

// log(1 + e^v) without overflow.
__device__ __forceinline__ float softplus_f(float v)
{
    return v > 20.0f ? v + log1pf(expf(-v)) : log1pf(expf(v));
}

// Eight consecutive elements as floats: one 16-byte load for bf16, two for fp32.
__device__ __forceinline__ void load8(const bf16* p, float (&v)[8])
{
    const uint4 r = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; i++) {
        v[2 * i] = __uint_as_float(w[i] << 16);
        v[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}
__device__ __forceinline__ void load8(const float* p, float (&v)[8])
{
    const float4 a = reinterpret_cast<const float4*>(p)[0];
    const float4 b = reinterpret_cast<const float4*>(p)[1];
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
}
__device__ __forceinline__ void store8(bf16* p, const float (&v)[8])
{
    uint4 r;
    uint32_t w[4];
#pragma unroll
    for (int i = 0; i < 4; i++) {
        const __nv_bfloat162 t = __floats2bfloat162_rn(v[2 * i], v[2 * i + 1]);
        w[i] = *reinterpret_cast<const uint32_t*>(&t);
    }
    r.x = w[0]; r.y = w[1]; r.z = w[2]; r.w = w[3];
    *reinterpret_cast<uint4*>(p) = r;
}
__device__ __forceinline__ void store8(float* p, const float (&v)[8])
{
    reinterpret_cast<float4*>(p)[0] = make_float4(v[0], v[1], v[2], v[3]);
    reinterpret_cast<float4*>(p)[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// 1 when seq[r] differs from seq[r-1] (r > 0): a packed-document boundary.
__device__ __forceinline__ int is_boundary(const int32_t* seq_row, int64_t r)
{
    return (seq_row != nullptr && r > 0) ? (seq_row[r] != seq_row[r - 1]) : 0;
}

// Real tokens of row b of a ragged batch (lengths null: every row is L long);
// lengths are clamped to [0, L].  Padding tokens after them carry dt = 0 and
// no document boundary, so the state passes them unchanged, and their outputs
// are written as +0.0.
__device__ __forceinline__ int row_length(const int32_t* lengths, int b, int L)
{
    if (lengths == nullptr) return L;
    const int v = lengths[b];
    return v < 0 ? 0 : (v > L ? L : v);
}

}  // namespace ssd
