// wkv7_forward_timemix: the forward with the time-mix block's output epilogue
// (the current-token term, the per-head normalisation and the gate; Paper
// Review: RWKV-7 "Goose", section "The approach"; the formula is EpiArgs's in
// common.cuh).
//
//  - Chunked form (bf16 inputs): the epilogue is part of the chunked kernel
//    (the current-token term on the diagonal of L_rk, the norm and the gate in
//    place of its y store), for one pass and for sequence segments alike.
//  - Sequential scan: the scan writes an fp32 y into the caller's workspace,
//    then timemix_epilogue_kernel maps it to z, one warp per head-token row.
#include "common.cuh"

namespace wkv7 {
namespace {

__device__ __forceinline__ float2 load2(const float *p) { return *reinterpret_cast<const float2 *>(p); }
__device__ __forceinline__ float2 load2(const __nv_bfloat16 *p) {
    const uint32_t u = *reinterpret_cast<const uint32_t *>(p);
    return make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xffff0000u));
}
__device__ __forceinline__ void store2(float *p, float2 x) { *reinterpret_cast<float2 *>(p) = x; }
__device__ __forceinline__ void store2(__nv_bfloat16 *p, float2 x) {
    *reinterpret_cast<__nv_bfloat162 *>(p) = __floats2bfloat162_rn(x.x, x.y);
}

__device__ __forceinline__ float warp_sum(float x) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) x += __shfl_xor_sync(0xffffffffu, x, o);
    return x;
}

constexpr int kEpiWarps = 8;

// z for `rows` head-token rows of [B, T, H, 64]; warp -> row, lane -> channels
// 2 lane, 2 lane + 1.  fp32 arithmetic, sums over the row by xor-shuffles.
template <typename InT, typename OutT>
__global__ void __launch_bounds__(32 * kEpiWarps)
timemix_epilogue_kernel(long long rows, int H, const float *__restrict__ y, const InT *__restrict__ r,
                        const InT *__restrict__ k, const InT *__restrict__ v, const float *__restrict__ rho,
                        const float *__restrict__ gamma, const float *__restrict__ beta, const InT *__restrict__ g,
                        float eps, OutT *__restrict__ z) {
    const long long row = (long long)blockIdx.x * kEpiWarps + (threadIdx.x >> 5);
    if (row >= rows) return;
    const int lane = threadIdx.x & 31, h = (int)(row % H), c = 2 * lane;
    const size_t off = (size_t)row * kN + c, po = (size_t)h * kN + c;
    const float2 rv = load2(r + off), kv = load2(k + off), vv = load2(v + off), pr = load2(rho + po);
    const float u = warp_sum(rv.x * pr.x * kv.x + rv.y * pr.y * kv.y);      // current-token weight
    const float2 yv = load2(y + off);
    const float o0 = fmaf(u, vv.x, yv.x), o1 = fmaf(u, vv.y, yv.y);
    const float mu = warp_sum(o0 + o1) * (1.f / kN);
    const float d0 = o0 - mu, d1 = o1 - mu;
    const float inv = rsqrtf(warp_sum(d0 * d0 + d1 * d1) * (1.f / kN) + eps);
    const float2 gm = gamma ? load2(gamma + po) : make_float2(1.f, 1.f);
    const float2 bt = beta ? load2(beta + po) : make_float2(0.f, 0.f);
    const float2 gv = g ? load2(g + off) : make_float2(1.f, 1.f);
    store2(z + off, make_float2(fmaf(d0 * inv, gm.x, bt.x) * gv.x, fmaf(d1 * inv, gm.y, bt.y) * gv.y));
}

cudaError_t timemix_epilogue(long long rows, int H, wkv7_dtype in_dt, wkv7_dtype out_dt, const float *y,
                             const void *r, const void *k, const void *v, const EpiArgs &epi, void *z,
                             cudaStream_t st) {
    const unsigned blocks = (unsigned)((rows + kEpiWarps - 1) / kEpiWarps);
#define WKV7_EPI_LAUNCH(I, O)                                                                                     \
    timemix_epilogue_kernel<I, O><<<blocks, 32 * kEpiWarps, 0, st>>>(                                             \
        rows, H, y, (const I *)r, (const I *)k, (const I *)v, epi.rho, epi.gamma, epi.beta, (const I *)epi.g,     \
        epi.eps, (O *)z)
    using bf = __nv_bfloat16;
    if (in_dt == WKV7_F32 && out_dt == WKV7_F32) WKV7_EPI_LAUNCH(float, float);
    else if (in_dt == WKV7_F32) WKV7_EPI_LAUNCH(float, bf);
    else if (out_dt == WKV7_F32) WKV7_EPI_LAUNCH(bf, float);
    else WKV7_EPI_LAUNCH(bf, bf);
#undef WKV7_EPI_LAUNCH
    return cudaGetLastError();
}

}  // namespace
}  // namespace wkv7

extern "C" {

size_t wkv7_forward_timemix_workspace_size(int B, int T, int H, int N, wkv7_dtype in_dtype, wkv7_algo algo,
                                           int chunk_len) {
    using namespace wkv7;
    if (B <= 0 || T <= 0 || H <= 0 || N != kN || (in_dtype != WKV7_F32 && in_dtype != WKV7_BF16)) return 0;
    const int code = wkv7_forward_resolve_algo(T, in_dtype, algo);
    if (code == WKV7_ALGO_CHUNK) return wkv7_forward_workspace_size(B, T, H, N, in_dtype, algo, chunk_len);
    if (code == WKV7_ALGO_SEQ) return (size_t)B * T * H * kN * sizeof(float);       // the fp32 y
    return 0;
}

wkv7_status wkv7_forward_timemix(int B, int T, int H, int N, wkv7_dtype in_dt, wkv7_dtype out_dt, const void *r,
                                 const void *w, const void *k, const void *v, const void *a, const void *b,
                                 const float *s0, const float *rho, const float *gamma, const float *beta,
                                 const void *g, float eps, void *z, float *sT, wkv7_algo algo, int chunk_len,
                                 void *workspace, size_t workspace_bytes, cudaStream_t stream) {
    using namespace wkv7;
    auto al16 = [](const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; };
    if (!(eps >= 0.f) || eps > 3.0e38f) return WKV7_ERR_INVALID_ARG;        // rejects NaN and inf too
    if (rho == nullptr || !al16(rho) || !al16(gamma) || !al16(beta) || !al16(g)) return WKV7_ERR_INVALID_ARG;
    const wkv7_status ds = check_dims(B, T, H, N);
    if (ds != WKV7_OK) return ds;
    const int code = wkv7_forward_resolve_algo(T, in_dt, algo);
    if (code < 0 || (out_dt != WKV7_F32 && out_dt != WKV7_BF16)) return WKV7_ERR_INVALID_ARG;
    EpiArgs epi{rho, gamma, beta, g, eps};
    if (code == WKV7_ALGO_CHUNK || T == 0 || (size_t)B * H == 0)
        return forward_impl(B, T, H, N, in_dt, out_dt, r, w, k, v, a, b, s0, z, sT, algo, chunk_len, workspace,
                            workspace_bytes, stream, nullptr, epi);
    // sequential scan: y in fp32 into the workspace, then the epilogue pass
    const size_t need = (size_t)B * T * H * kN * sizeof(float);
    if (workspace == nullptr || !al16(workspace) || workspace_bytes < need || !al16(z) || z == nullptr)
        return WKV7_ERR_INVALID_ARG;
    float *y = static_cast<float *>(workspace);
    const wkv7_status s = wkv7_forward(B, T, H, N, in_dt, WKV7_F32, r, w, k, v, a, b, s0, y, sT, algo, chunk_len,
                                       nullptr, 0, stream);
    if (s != WKV7_OK) return s;
    return timemix_epilogue((long long)B * T * H, H, in_dt, out_dt, y, r, k, v, epi, z, stream) == cudaSuccess
               ? WKV7_OK
               : WKV7_ERR_CUDA;
}

}  // extern "C"
