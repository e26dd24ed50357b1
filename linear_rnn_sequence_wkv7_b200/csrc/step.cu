// Decode step (T = 1): one token of the WKV7 recurrence for every (b, h), with
// the fp32 state updated in place.  A decode step costs constant time and
// memory per token (RWKV-7 "Goose" with Expressive Dynamic State Evolution,
// abstract); on B200 it is bound by the state's read-modify-write in HBM.
//
// Mapping: one CTA per (b, h) head, 256 threads.  Sixteen consecutive lanes
// own one 256-byte state row (lane l holds columns 4l..4l+3 as a float4), a
// warp covers two rows per pass and each thread handles the rows
// i = slot + 16 u (u = 0..3), whose four float4 loads are issued together so
// 64 bytes per thread are in flight.  The two per-row dot products are
// 4-term in-thread sums plus four xor-shuffle steps inside the 16-lane group.
// The token's vectors (5 x 4 elements per lane, plus v per row) are read
// straight from global memory; all rows of the head share them through L1.
#include "common.cuh"

namespace wkv7 {

template <typename InT, typename OutT>
__global__ void __launch_bounds__(256)
step_kernel(const InT *__restrict__ r, const InT *__restrict__ w, const InT *__restrict__ k,
            const InT *__restrict__ v, const InT *__restrict__ a, const InT *__restrict__ b,
            float *__restrict__ state, OutT *__restrict__ y) {
    constexpr int ROWS_PER_THREAD = 4;
    const int head = blockIdx.x;               // flattened (b, h)
    const int lane16 = threadIdx.x & 15;
    const int slot = threadIdx.x >> 4;         // 0..15
    const size_t vbase = (size_t)head * kN;
    float *S = state + (size_t)head * kN * kN;

    float4 s4[ROWS_PER_THREAD];
#pragma unroll
    for (int u = 0; u < ROWS_PER_THREAD; ++u)
        s4[u] = __ldcs(reinterpret_cast<const float4 *>(S + (size_t)(slot + 16 * u) * kN + 4 * lane16));

    const float4 a4 = load4(a + vbase + 4 * lane16);
    const float4 w4 = load4(w + vbase + 4 * lane16);
    const float4 b4 = load4(b + vbase + 4 * lane16);
    const float4 k4 = load4(k + vbase + 4 * lane16);
    const float4 r4 = load4(r + vbase + 4 * lane16);
    float vi[ROWS_PER_THREAD];
#pragma unroll
    for (int u = 0; u < ROWS_PER_THREAD; ++u) vi[u] = to_f32(v[vbase + slot + 16 * u]);

    float p[ROWS_PER_THREAD];
#pragma unroll
    for (int u = 0; u < ROWS_PER_THREAD; ++u)
        p[u] = fmaf(s4[u].x, a4.x, fmaf(s4[u].y, a4.y, fmaf(s4[u].z, a4.z, s4[u].w * a4.w)));
#pragma unroll
    for (int off = 1; off < 16; off <<= 1)
#pragma unroll
        for (int u = 0; u < ROWS_PER_THREAD; ++u) p[u] += __shfl_xor_sync(0xffffffffu, p[u], off);

    float yv[ROWS_PER_THREAD];
#pragma unroll
    for (int u = 0; u < ROWS_PER_THREAD; ++u) {
        float4 s = s4[u];
        s.x = fmaf(s.x, w4.x, fmaf(p[u], b4.x, vi[u] * k4.x));
        s.y = fmaf(s.y, w4.y, fmaf(p[u], b4.y, vi[u] * k4.y));
        s.z = fmaf(s.z, w4.z, fmaf(p[u], b4.z, vi[u] * k4.z));
        s.w = fmaf(s.w, w4.w, fmaf(p[u], b4.w, vi[u] * k4.w));
        __stcs(reinterpret_cast<float4 *>(S + (size_t)(slot + 16 * u) * kN + 4 * lane16), s);
        yv[u] = fmaf(s.x, r4.x, fmaf(s.y, r4.y, fmaf(s.z, r4.z, s.w * r4.w)));
    }
#pragma unroll
    for (int off = 1; off < 16; off <<= 1)
#pragma unroll
        for (int u = 0; u < ROWS_PER_THREAD; ++u) yv[u] += __shfl_xor_sync(0xffffffffu, yv[u], off);
#pragma unroll
    for (int u = 0; u < ROWS_PER_THREAD; ++u)
        if (lane16 == u) y[vbase + slot + 16 * u] = from_f32<OutT>(yv[u]);
}

cudaError_t step(int B, int H, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r, const void *w,
                 const void *k, const void *v, const void *a, const void *b, float *state, void *y,
                 cudaStream_t st) {
    dim3 grid((unsigned)(B * H));
#define WKV7_STEP_LAUNCH(I, O)                                                                          \
    step_kernel<I, O><<<grid, 256, 0, st>>>((const I *)r, (const I *)w, (const I *)k, (const I *)v,     \
                                            (const I *)a, (const I *)b, state, (O *)y)
    if (in_dt == WKV7_F32 && y_dt == WKV7_F32) WKV7_STEP_LAUNCH(float, float);
    else if (in_dt == WKV7_F32) WKV7_STEP_LAUNCH(float, __nv_bfloat16);
    else if (y_dt == WKV7_F32) WKV7_STEP_LAUNCH(__nv_bfloat16, float);
    else WKV7_STEP_LAUNCH(__nv_bfloat16, __nv_bfloat16);
#undef WKV7_STEP_LAUNCH
    return cudaGetLastError();
}

}  // namespace wkv7
