// Shared device helpers of the WKV7 CUDA library (sm_100a).
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "wkv7.h"

namespace wkv7 {

constexpr int kN = 64;  // head size the kernels implement

// A 32-token chunk's transition [M^T; Q] (S_out = S_in M + E, y_t = S_in q_t +
// terms without S_in; row m of M^T is column m of M, row t of Q is q_t) as the
// checkpoint pass of the chunked forward exports it for the backward: the bf16
// hi image of a 96 x 64 tile in core-matrix layout (rows m = 0..63, then t),
// then the lo image; counted in 16-byte words.
constexpr int kMqChunkVec = 2 * 96 * kN * 2 / 16;

// Sticky device-side status word (one per device): kernels that detect a
// bounded wait running out or an out-of-domain chunk set it with atomicMax;
// wkv7_get_device_status reads and clears it.  Defined here because the
// library is compiled as a single translation unit (csrc/libwkv7.cu).
__device__ int g_device_status = 0;

__device__ __forceinline__ void raise_status(int code) { atomicMax(&g_device_status, code); }

// Optional output epilogue of the time-mix block (Paper Review: RWKV-7
// "Goose", section "The approach": the receptance reads the state, the block
// also attends to the current token without storing it, and the output is
// normalised per head and gated).  With rho set, y_t is replaced by
//     o_t = S_t r_t + (sum_j r_t[j] rho[j] k_t[j]) v_t
//     z_t = g_t * (gamma * (o_t - mean(o_t)) / sqrt(var(o_t) + eps) + beta)
// (mean and population variance over the head's N channels; gamma, beta, g
// default to 1, 0, 1).  The chunked kernel applies it in place of its y
// store and adds the current-token term to the diagonal of the chunk's L_rk
// (token t's own write already reaches y_t through r_t . k_t, so the term only
// reweights it): it never enters the state.  The sequential path runs it as a
// separate pass over an fp32 y.
struct EpiArgs {
    const float *rho;             // [H][64] or null: no epilogue, plain y
    const float *gamma, *beta;    // [H][64] or null
    const void *g;                // [B][T][H][64] of the input dtype, or null
    float eps;
};

// ---- element load / store ---------------------------------------------------

__device__ __forceinline__ float to_f32(float x) { return x; }
__device__ __forceinline__ float to_f32(__nv_bfloat16 x) { return __bfloat162float(x); }

template <typename T> __device__ __forceinline__ T from_f32(float x);
template <> __device__ __forceinline__ float from_f32<float>(float x) { return x; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float x) {
    return __float2bfloat16_rn(x);
}

// Load 4 consecutive elements (16-byte aligned for fp32, 8-byte for bf16) as float4.
__device__ __forceinline__ float4 load4(const float *p) { return *reinterpret_cast<const float4 *>(p); }
__device__ __forceinline__ float4 load4(const __nv_bfloat16 *p) {
    uint2 u = *reinterpret_cast<const uint2 *>(p);
    float4 f;
    f.x = __uint_as_float(u.x << 16);
    f.y = __uint_as_float(u.x & 0xffff0000u);
    f.z = __uint_as_float(u.y << 16);
    f.w = __uint_as_float(u.y & 0xffff0000u);
    return f;
}

__device__ __forceinline__ void store4(float *p, float4 v) { *reinterpret_cast<float4 *>(p) = v; }
__device__ __forceinline__ void store4(__nv_bfloat16 *p, float4 v) {
    __nv_bfloat162 lo = __floats2bfloat162_rn(v.x, v.y);
    __nv_bfloat162 hi = __floats2bfloat162_rn(v.z, v.w);
    uint2 u;
    u.x = *reinterpret_cast<uint32_t *>(&lo);
    u.y = *reinterpret_cast<uint32_t *>(&hi);
    *reinterpret_cast<uint2 *>(p) = u;
}

// ---- cp.async (16-byte, L2 only) ---------------------------------------------

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}
__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gmem_src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(smem_u32(smem_dst)), "l"(gmem_src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;\n" ::"n"(N) : "memory");
}

}  // namespace wkv7
