// Sequential-scan WKV7 forward (token by token, state on chip).
//
// Per head, row i of the state evolves independently given the token's
// shared vectors (the "diagonal plus rank one" transition of RWKV-7: Paper
// Review: RWKV-7 "Goose", sections "Architecture" and "The approach"):
//     p = S[i,:] . a_t ;  S[i,j] = S[i,j] w_t[j] + p b_t[j] + v_t[i] k_t[j] ;
//     y_t[i] = S[i,:] . r_t
//
// Mapping: a CTA owns RB rows of one (b, h) state.  Four consecutive lanes
// share a row group of RPT rows; lane q holds the 16 columns
// j = 16 m + 4 q + e (m, e in 0..3) of each of its rows in registers, so the
// two dot products per token are 16-term in-thread sums plus two xor-shuffle
// steps, and the update is 3 FP32 instructions per element.  The token
// vectors are streamed through shared memory in double-buffered tiles of TT
// tokens: with TMA, one thread issues a tile load per tensor ([TT tokens] x
// [64 channels] of the (b, h) slice, rows past T filled with zeros), each
// stage completing on its own mbarrier; otherwise every thread issues 16-byte
// cp.async copies.  bf16 tiles are converted to fp32 once per CTA, and every
// lane reads them as broadcast float4s (the interleaved column assignment
// keeps the 4 lanes of a row group on distinct banks).
//
// CKPT mode writes the state before every CK-th token to a checkpoint buffer
// (the backward's first pass, without y; the training forward, with y).
#include <cuda.h>
#include <cudaTypedefs.h>

#include "umma.cuh"

namespace wkv7 {

// TMA descriptors of the six token tensors r w k v a b, each seen as a 3D
// array {x: H * 64 channels, y: T tokens, z: B}
struct SeqMaps {
    CUtensorMap m[6];
};

__device__ __forceinline__ void seq_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}

// one box of a 3D tensor map into shared memory (no multicast), completing
// on the mbarrier at `bar`
__device__ __forceinline__ void seq_tma_load(uint32_t dst, const CUtensorMap *map, int x, int y, int z, uint32_t bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3, %4}], [%5];"
        ::"r"(dst), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y), "r"(z), "r"(bar)
        : "memory");
}

template <typename InT, typename OutT, int RPT, int RB, int TT, bool CKPT, bool YOUT, bool TMA>
__global__ void __launch_bounds__((RB / RPT) * 4)
fwd_seq_kernel(int T, int H, const __grid_constant__ SeqMaps maps, const InT *__restrict__ r,
               const InT *__restrict__ w, const InT *__restrict__ k, const InT *__restrict__ v,
               const InT *__restrict__ a, const InT *__restrict__ b, const float *s0, OutT *__restrict__ y,
               float *sT, float *__restrict__ ckpt, int CK, long long wait_limit) {
    constexpr int NT = (RB / RPT) * 4;
    constexpr int NTEN = 6;                          // r w k v a b
    constexpr uint32_t TILE_BYTES = TT * kN * sizeof(InT);        // one tensor's tile
    constexpr bool kConvert = !std::is_same<InT, float>::value;

    extern __shared__ __align__(128) unsigned char smem_raw[];
    InT *raw = reinterpret_cast<InT *>(smem_raw);                 // [2][NTEN][TT][kN]
    float *f32buf = kConvert ? reinterpret_cast<float *>(smem_raw + 2 * NTEN * TILE_BYTES)
                             : nullptr;                           // [NTEN][TT][kN]
    const uint32_t bar0 = smem_u32(smem_raw + 2 * NTEN * TILE_BYTES +
                                   (kConvert ? NTEN * TT * kN * sizeof(float) : 0));   // 2 mbarriers
    const int tid = threadIdx.x;
    const int q = tid & 3;
    const int rg = tid >> 2;
    const int blocks_per_head = kN / RB;
    const int h = blockIdx.x / blocks_per_head;
    const int row0 = (blockIdx.x % blocks_per_head) * RB + rg * RPT;
    const int bb = blockIdx.y;
    const size_t tok_stride = (size_t)H * kN;                     // between consecutive t
    const size_t base = ((size_t)bb * T * H + h) * kN;            // (bb, t=0, h, 0)
    const size_t st_base = ((size_t)bb * H + h) * kN * kN;

    if constexpr (TMA) {                                          // one mbarrier per tile stage
        if (tid == 0) {
            umma::mbar_init(bar0, 1);
            umma::mbar_init(bar0 + 8, 1);
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncthreads();
    }

    float S[RPT][16];
#pragma unroll
    for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float4 s4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (s0) s4 = load4(s0 + st_base + (size_t)(row0 + rr) * kN + 16 * m + 4 * q);
            S[rr][4 * m + 0] = s4.x;
            S[rr][4 * m + 1] = s4.y;
            S[rr][4 * m + 2] = s4.z;
            S[rr][4 * m + 3] = s4.w;
        }

    const int ntiles = (T + TT - 1) / TT;
    // tile `tile` into stage `stage`: with TMA, thread 0 loads the six
    // tensors' boxes at x = 64 h (128-byte aligned), y = first token, z = b;
    // else all threads copy the tile's rows that lie before T
    const InT *src[NTEN] = {r, w, k, v, a, b};
    auto issue_tile = [&](int tile, int stage) {
        if constexpr (TMA) {
            if (tid != 0) return;
            const uint32_t bar = bar0 + 8u * (uint32_t)stage;
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");   // the stage's last generic reads
            seq_expect_tx(bar, NTEN * TILE_BYTES);
#pragma unroll
            for (int ten = 0; ten < NTEN; ++ten)
                seq_tma_load(smem_u32(raw + ((size_t)stage * NTEN + ten) * TT * kN), &maps.m[ten], h * kN, tile * TT,
                             bb, bar);
        } else {
            constexpr int VEC = 16 / sizeof(InT), CPV = kN / VEC;       // 16-byte chunks per N-vector
            const int t0 = tile * TT;
            for (int c = tid; c < TT * NTEN * CPV; c += NT) {
                const int ten = c / (TT * CPV), rem = c % (TT * CPV), tt = rem / CPV, ch = rem % CPV;
                if (t0 + tt < T)
                    cp_async16(raw + (((size_t)stage * NTEN + ten) * TT + tt) * kN + ch * VEC,
                               src[ten] + base + (size_t)(t0 + tt) * tok_stride + ch * VEC);
            }
            cp_async_commit();
        }
    };

    if (ntiles > 0) issue_tile(0, 0);
    for (int it = 0; it < ntiles; ++it) {
        const int stage = it & 1;
        const int t0 = it * TT;
        // the tile's bytes have landed: with TMA phase it / 2 of its stage's
        // mbarrier (bounded; polled with test_wait), else this thread's copies
        bool late = false;
        if constexpr (TMA)
            late = !umma::mbar_spin(bar0 + 8u * (uint32_t)stage, (uint32_t)(it >> 1) & 1u, wait_limit);
        else
            cp_async_wait<0>();
        if (__syncthreads_or(late)) {
            // a tile did not arrive within the limit: report it, give the one
            // copy in flight (this tile's; the next is not issued yet) a
            // bounded time to land, and stop without writing y or sT
            if (tid == 0) {
                raise_status(WKV7_ERR_TIMEOUT);
                umma::mbar_wait(bar0 + 8u * (uint32_t)stage, (uint32_t)(it >> 1) & 1u, 200000000LL);
            }
            return;
        }
        const float *buf;
        if constexpr (kConvert) {
            const InT *rs = raw + (size_t)stage * NTEN * TT * kN;
            for (int e = tid * 4; e < NTEN * TT * kN; e += NT * 4) store4(f32buf + e, load4(rs + e));
            __syncthreads();
            buf = f32buf;
        } else {
            buf = reinterpret_cast<const float *>(raw) + (size_t)stage * NTEN * TT * kN;
        }
        if (it + 1 < ntiles) issue_tile(it + 1, stage ^ 1);

        if constexpr (CKPT) {
            if (t0 % CK == 0) {
                float *dst = ckpt + (((size_t)bb * H + h) * ((T + CK - 1) / CK) + t0 / CK) * kN * kN;
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
                    for (int m = 0; m < 4; ++m)
                        store4(dst + (size_t)(row0 + rr) * kN + 16 * m + 4 * q,
                               make_float4(S[rr][4 * m], S[rr][4 * m + 1], S[rr][4 * m + 2], S[rr][4 * m + 3]));
            }
        }

        const int tt_end = min(TT, T - t0);
        for (int tt = 0; tt < tt_end; ++tt) {
            const float *rv = buf + (0 * TT + tt) * kN;
            const float *wv = buf + (1 * TT + tt) * kN;
            const float *kv = buf + (2 * TT + tt) * kN;
            const float *vv = buf + (3 * TT + tt) * kN;
            const float *av = buf + (4 * TT + tt) * kN;
            const float *bv = buf + (5 * TT + tt) * kN;

            // p = S_{t-1}[i,:] . a_t, in packed fp32 pairs (fma.rn.f32x2): two
            // partial sums per row, half the FP instructions
            float p[RPT];
            {
                float2 p2[RPT];
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) p2[rr] = make_float2(0.f, 0.f);
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(av + 16 * m + 4 * q);
                    const float2 alo = make_float2(a4.x, a4.y), ahi = make_float2(a4.z, a4.w);
#pragma unroll
                    for (int rr = 0; rr < RPT; ++rr) {
                        p2[rr] = __ffma2_rn(make_float2(S[rr][4 * m + 0], S[rr][4 * m + 1]), alo, p2[rr]);
                        p2[rr] = __ffma2_rn(make_float2(S[rr][4 * m + 2], S[rr][4 * m + 3]), ahi, p2[rr]);
                    }
                }
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) p[rr] = p2[rr].x + p2[rr].y;
            }
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) {
                p[rr] += __shfl_xor_sync(0xffffffffu, p[rr], 1);
                p[rr] += __shfl_xor_sync(0xffffffffu, p[rr], 2);
            }
            float vi[RPT];
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) vi[rr] = vv[row0 + rr];

            // S = S * w + p b + v k ;  y = S . r   (packed fp32 pairs, the same
            // per-element rounding for S; y summed as two partial sums)
            float yacc[RPT];
            float2 y2[RPT];
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) y2[rr] = make_float2(0.f, 0.f);
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 w4 = *reinterpret_cast<const float4 *>(wv + 16 * m + 4 * q);
                const float4 b4 = *reinterpret_cast<const float4 *>(bv + 16 * m + 4 * q);
                const float4 k4 = *reinterpret_cast<const float4 *>(kv + 16 * m + 4 * q);
                const float4 r4 = *reinterpret_cast<const float4 *>(rv + 16 * m + 4 * q);
                const float2 wj[2] = {make_float2(w4.x, w4.y), make_float2(w4.z, w4.w)};
                const float2 bj[2] = {make_float2(b4.x, b4.y), make_float2(b4.z, b4.w)};
                const float2 kj[2] = {make_float2(k4.x, k4.y), make_float2(k4.z, k4.w)};
                const float2 rj[2] = {make_float2(r4.x, r4.y), make_float2(r4.z, r4.w)};
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) {
                    const float2 pp = make_float2(p[rr], p[rr]), vv2 = make_float2(vi[rr], vi[rr]);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float2 s = make_float2(S[rr][4 * m + 2 * e], S[rr][4 * m + 2 * e + 1]);
                        s = __ffma2_rn(s, wj[e], __ffma2_rn(pp, bj[e], __fmul2_rn(vv2, kj[e])));
                        S[rr][4 * m + 2 * e] = s.x;
                        S[rr][4 * m + 2 * e + 1] = s.y;
                        if constexpr (YOUT) y2[rr] = __ffma2_rn(s, rj[e], y2[rr]);
                    }
                }
            }
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) yacc[rr] = y2[rr].x + y2[rr].y;
            if constexpr (YOUT) {
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr) {
                    yacc[rr] += __shfl_xor_sync(0xffffffffu, yacc[rr], 1);
                    yacc[rr] += __shfl_xor_sync(0xffffffffu, yacc[rr], 2);
                }
                OutT *yrow = y + base + (size_t)(t0 + tt) * tok_stride + row0;
#pragma unroll
                for (int rr = 0; rr < RPT; ++rr)
                    if (q == (rr & 3)) yrow[rr] = from_f32<OutT>(yacc[rr]);
            }
        }
    }

    if (sT) {
        // Every CTA read its own rows of s0 before its first tile, so writing
        // sT here is safe even when sT aliases s0.
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
            for (int m = 0; m < 4; ++m)
                store4(sT + st_base + (size_t)(row0 + rr) * kN + 16 * m + 4 * q,
                       make_float4(S[rr][4 * m], S[rr][4 * m + 1], S[rr][4 * m + 2], S[rr][4 * m + 3]));
    }
}

// cuTensorMapEncodeTiled, looked up in the driver once (no link-time
// dependency on the driver library)
static PFN_cuTensorMapEncodeTiled_v12000 seq_encode_fn() {
    static const PFN_cuTensorMapEncodeTiled_v12000 fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return (PFN_cuTensorMapEncodeTiled_v12000) nullptr;
        return reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
    }();
    return fn;
}

// The six token tensors [B, T, H, 64] as 3D maps {H * 64, T, B} with boxes of
// {64, TT, 1}: a (b, h) slice of TT tokens, rows past T read as zeros.  Base
// addresses are 16-byte aligned (the API checks every pointer) and the row
// strides are multiples of 128 bytes.
template <typename InT, int TT>
static cudaError_t seq_maps(int B, int T, int H, const void *const src[6], SeqMaps &maps) {
    const PFN_cuTensorMapEncodeTiled_v12000 encode = seq_encode_fn();
    if (!encode) return cudaErrorNotSupported;
    const CUtensorMapDataType dt =
        std::is_same<InT, float>::value ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16;
    const cuuint64_t dims[3] = {(cuuint64_t)H * kN, (cuuint64_t)T, (cuuint64_t)B};
    const cuuint64_t strides[2] = {(cuuint64_t)H * kN * sizeof(InT), (cuuint64_t)T * H * kN * sizeof(InT)};
    const cuuint32_t box[3] = {(cuuint32_t)kN, (cuuint32_t)TT, 1u};
    const cuuint32_t estr[3] = {1u, 1u, 1u};
    for (int x = 0; x < 6; ++x) {
        const CUresult res = encode(&maps.m[x], dt, 3, const_cast<void *>(src[x]), dims, strides, box, estr,
                                    CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                                    CU_TENSOR_MAP_L2_PROMOTION_L2_128B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
        if (res != CUDA_SUCCESS) return cudaErrorInvalidValue;
    }
    return cudaSuccess;
}

template <typename InT, typename OutT, int RPT, int RB, int TT, bool CKPT, bool YOUT, bool TMA>
static cudaError_t launch_fwd_seq(int B, int T, int H, const void *r, const void *w, const void *k,
                                  const void *v, const void *a, const void *b, const float *s0, void *y,
                                  float *sT, float *ckpt, int CK, long long wait_limit, cudaStream_t st) {
    constexpr int NT = (RB / RPT) * 4;
    size_t smem = 2 * 6 * TT * kN * sizeof(InT);
    if (!std::is_same<InT, float>::value) smem += 6 * TT * kN * sizeof(float);
    smem += 16;                                      // two mbarriers
    SeqMaps maps{};
    const void *src[6] = {r, w, k, v, a, b};
    cudaError_t e = TMA ? seq_maps<InT, TT>(B, T, H, src, maps) : cudaSuccess;
    if (e != cudaSuccess) return e;
    auto kern = fwd_seq_kernel<InT, OutT, RPT, RB, TT, CKPT, YOUT, TMA>;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    dim3 grid(H * (kN / RB), B);
    kern<<<grid, NT, smem, st>>>(T, H, maps, (const InT *)r, (const InT *)w, (const InT *)k, (const InT *)v,
                                 (const InT *)a, (const InT *)b, s0, (OutT *)y, sT, ckpt, CK, wait_limit);
    return cudaGetLastError();
}

// Layout of the scan: with more heads than SMs, one CTA per head with four
// rows per thread and 32-token tiles loaded by TMA (fewer loads and
// conversions of the token vectors per row: 1.87 vs 2.29 ms at B=8, T=4096,
// H=32, bf16, of which TMA instead of cp.async 0.013 ms); otherwise two CTAs
// per head with two rows per thread and 16-token tiles by cp.async, which
// keeps more SMs busy (1.69 vs 1.85 ms at B=2; TMA tiles measured 1.89 ms
// there).
template <typename InT, typename OutT, bool CKPT, bool YOUT = !CKPT>
static cudaError_t dispatch_fwd_seq(int B, int T, int H, const void *r, const void *w, const void *k, const void *v,
                                    const void *a, const void *b, const float *s0, void *y, float *sT, float *ckpt,
                                    int CK, long long lim, cudaStream_t st) {
    if ((long long)B * H > 148 && (!CKPT || CK % 32 == 0))   // checkpoints fall on tile starts
        return launch_fwd_seq<InT, OutT, 4, 64, 32, CKPT, YOUT, true>(B, T, H, r, w, k, v, a, b, s0, y, sT, ckpt, CK,
                                                                      lim, st);
    return launch_fwd_seq<InT, OutT, 2, 32, 16, CKPT, YOUT, false>(B, T, H, r, w, k, v, a, b, s0, y, sT, ckpt, CK, lim,
                                                                   st);
}

// Host entry used by the API layer.
cudaError_t fwd_seq(int B, int T, int H, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r,
                    const void *w, const void *k, const void *v, const void *a, const void *b,
                    const float *s0, void *y, float *sT, long long lim, cudaStream_t st) {
    if (in_dt == WKV7_F32 && y_dt == WKV7_F32)
        return dispatch_fwd_seq<float, float, false>(B, T, H, r, w, k, v, a, b, s0, y, sT, nullptr, 0, lim, st);
    if (in_dt == WKV7_F32 && y_dt == WKV7_BF16)
        return dispatch_fwd_seq<float, __nv_bfloat16, false>(B, T, H, r, w, k, v, a, b, s0, y, sT, nullptr, 0, lim, st);
    if (in_dt == WKV7_BF16 && y_dt == WKV7_F32)
        return dispatch_fwd_seq<__nv_bfloat16, float, false>(B, T, H, r, w, k, v, a, b, s0, y, sT, nullptr, 0, lim, st);
    return dispatch_fwd_seq<__nv_bfloat16, __nv_bfloat16, false>(B, T, H, r, w, k, v, a, b, s0, y, sT, nullptr, 0, lim, st);
}

// State checkpoints every CK tokens (CK a multiple of 16; they are written at
// the start of a token tile), and the final state
// when sT is given: ckpt[b][h][c] holds
// the state before token c * CK.  Used by the backward's first pass.
cudaError_t fwd_checkpoints(int B, int T, int H, wkv7_dtype in_dt, const void *r, const void *w,
                            const void *k, const void *v, const void *a, const void *b, const float *s0,
                            float *ckpt, int CK, float *sT, long long lim, cudaStream_t st) {
    if (in_dt == WKV7_F32)
        return dispatch_fwd_seq<float, float, true>(B, T, H, r, w, k, v, a, b, s0, nullptr, sT, ckpt, CK, lim, st);
    return dispatch_fwd_seq<__nv_bfloat16, float, true>(B, T, H, r, w, k, v, a, b, s0, nullptr, sT, ckpt, CK, lim, st);
}

// The forward with y and the state checkpoints every CK tokens (the training
// forward: the backward then skips its own checkpoint pass).
cudaError_t fwd_seq_train(int B, int T, int H, wkv7_dtype in_dt, wkv7_dtype y_dt, const void *r, const void *w,
                          const void *k, const void *v, const void *a, const void *b, const float *s0, void *y,
                          float *sT, float *ckpt, int CK, long long lim, cudaStream_t st) {
    if (in_dt == WKV7_F32 && y_dt == WKV7_F32)
        return dispatch_fwd_seq<float, float, true, true>(B, T, H, r, w, k, v, a, b, s0, y, sT, ckpt, CK, lim, st);
    if (in_dt == WKV7_F32 && y_dt == WKV7_BF16)
        return dispatch_fwd_seq<float, __nv_bfloat16, true, true>(B, T, H, r, w, k, v, a, b, s0, y, sT, ckpt, CK, lim, st);
    if (in_dt == WKV7_BF16 && y_dt == WKV7_F32)
        return dispatch_fwd_seq<__nv_bfloat16, float, true, true>(B, T, H, r, w, k, v, a, b, s0, y, sT, ckpt, CK, lim, st);
    return dispatch_fwd_seq<__nv_bfloat16, __nv_bfloat16, true, true>(B, T, H, r, w, k, v, a, b, s0, y, sT, ckpt, CK,
                                                                       lim, st);
}

}  // namespace wkv7
