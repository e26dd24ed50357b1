// Reverse-time WKV7 backward.
//
// Gradient of L = sum(dy * y) + sum(dsT * sT).  With g = dL/dS_t for one state
// row i (reverse time, t = T-1 .. 0):
//     g      += dy_t[i] r_t
//     dr_t   += dy_t[i] S_t[i,:]         dv_t[i] = g . k_t
//     dk_t   += v_t[i] g                 dw_t   += S_{t-1}[i,:] * g
//     db_t   += p_t[i] g   (p_t[i] = S_{t-1}[i,:] . a_t)
//     dp      = g . b_t                  da_t   += dp S_{t-1}[i,:]
//     g       = g * w_t + dp a_t         (dL/dS_{t-1})
// and ds0 = g at the end.  dr, dk, dw, db, da are sums over the rows of the
// head; dv and dp are per-row dot products.
//
// Pass A (fwd_checkpoints, in fwd_seq.cu) stores the state before every
// CK-th token.  Pass B (this file): one CTA per (b, h), 4 lanes per row and
// RPT rows per thread exactly as in the sequential forward.  For each chunk,
// last first: recompute the chunk's states from its checkpoint, writing each
// thread's own pre-token state slice to a private history in global scratch
// (CK x 16 KB per head, small enough to stay in L2) and p_t to shared memory;
// then sweep the chunk backwards.  Row sums are reduced by a transposed
// reduce-scatter across the warp's 8 row groups (each lane ends with 10 of
// the warp's 320 column sums) and added into a per-chunk shared accumulator
// with shared-memory atomics; the accumulator is written out once per chunk.
// Inputs and the next checkpoint are prefetched with cp.async one chunk
// ahead.
#include "common.cuh"

namespace wkv7 {

namespace {

constexpr int kRPT = 2;
constexpr int kNT = (kN / kRPT) * 4;   // 128 threads per head
constexpr int kNTEN = 7;               // r w k v a b dy
constexpr int kNRED = 5;               // dr dk dw db da

// Transposed reduce-scatter of X values across the lanes that differ in lane
// bit `bit`: afterwards the lane keeps X/2 sums (lower half if its bit is 0).
template <int X>
__device__ __forceinline__ void rs_step(float (&vals)[80], int bitmask) {
    const bool hi = (threadIdx.x & bitmask) != 0;
#pragma unroll
    for (int i = 0; i < X / 2; ++i) {
        const float lo_v = vals[i], hi_v = vals[X / 2 + i];
        const float send = hi ? lo_v : hi_v;
        const float keep = hi ? hi_v : lo_v;
        vals[i] = keep + __shfl_xor_sync(0xffffffffu, send, bitmask);
    }
}

}  // namespace

template <typename InT, typename GradT>
__global__ void __launch_bounds__(kNT)
bwd_seq_kernel(int T, int H, int CK, const InT *__restrict__ r, const InT *__restrict__ w,
               const InT *__restrict__ k, const InT *__restrict__ v, const InT *__restrict__ a,
               const InT *__restrict__ b, const InT *__restrict__ dy, const float *__restrict__ dsT,
               const float *__restrict__ ckpt, float4 *__restrict__ hist, GradT *__restrict__ dr,
               GradT *__restrict__ dw, GradT *__restrict__ dk, GradT *__restrict__ dv,
               GradT *__restrict__ da, GradT *__restrict__ db, float *__restrict__ ds0) {
    constexpr int VEC = 16 / sizeof(InT);
    constexpr int CPV = kN / VEC;   // 16-byte chunks per N-vector
    extern __shared__ __align__(16) unsigned char smem[];
    // layout: raw inputs [2][7][CK][64] InT | raw ckpt [2][64*64] f32 |
    //         fbuf [7][CK][64] f32 | acc [CK][5][64] f32 | p_s [CK][64] f32
    InT *raw = reinterpret_cast<InT *>(smem);
    float *ck_raw = reinterpret_cast<float *>(smem + 2 * kNTEN * CK * kN * sizeof(InT));
    float *fbuf = ck_raw + 2 * kN * kN;
    float *acc = fbuf + kNTEN * CK * kN;
    float *p_s = acc + CK * kNRED * kN;

    const int tid = threadIdx.x;
    const int q = tid & 3;
    const int rg = tid >> 2;
    const int row0 = rg * kRPT;
    const int head = blockIdx.x;   // b * H + h
    const int bb = head / H, h = head % H;
    const size_t tok_stride = (size_t)H * kN;
    const size_t base = ((size_t)bb * T * H + h) * kN;
    const size_t st_base = (size_t)head * kN * kN;
    const int nck = (T + CK - 1) / CK;
    const InT *src[kNTEN] = {r, w, k, v, a, b, dy};
    float4 *my_hist = hist + (size_t)head * CK * (kRPT * 4) * kNT;

    auto issue_chunk = [&](int c, int stage) {
        const int t0 = c * CK;
        const int L = min(CK, T - t0);
        for (int x = tid; x < kNTEN * CK * CPV; x += kNT) {
            const int ten = x / (CK * CPV);
            const int rem = x % (CK * CPV);
            const int tt = rem / CPV, ch = rem % CPV;
            if (tt < L)
                cp_async16(raw + (((size_t)stage * kNTEN + ten) * CK + tt) * kN + ch * VEC,
                           src[ten] + base + (size_t)(t0 + tt) * tok_stride + ch * VEC);
        }
        const float *cks = ckpt + ((size_t)head * nck + c) * kN * kN;
        for (int x = tid; x < kN * kN / 4; x += kNT) cp_async16(ck_raw + stage * kN * kN + 4 * x, cks + 4 * x);
        cp_async_commit();
    };

    float g[kRPT][16];
#pragma unroll
    for (int rr = 0; rr < kRPT; ++rr)
#pragma unroll
        for (int m = 0; m < 4; ++m) {
            float4 d4 = make_float4(0.f, 0.f, 0.f, 0.f);
            if (dsT) d4 = load4(dsT + st_base + (size_t)(row0 + rr) * kN + 16 * m + 4 * q);
            g[rr][4 * m] = d4.x; g[rr][4 * m + 1] = d4.y; g[rr][4 * m + 2] = d4.z; g[rr][4 * m + 3] = d4.w;
        }

    if (nck > 0) issue_chunk(nck - 1, 0);
    for (int c = nck - 1; c >= 0; --c) {
        const int stage = (nck - 1 - c) & 1;
        const int t0 = c * CK;
        const int L = min(CK, T - t0);
        cp_async_wait<0>();
        __syncthreads();
        {
            const InT *rs = raw + (size_t)stage * kNTEN * CK * kN;
            for (int e = tid * 4; e < kNTEN * CK * kN; e += kNT * 4) {
                const int tt = (e / kN) % CK;
                store4(fbuf + e, tt < L ? load4(rs + e) : make_float4(0.f, 0.f, 0.f, 0.f));
            }
            for (int e = tid; e < CK * kNRED * kN; e += kNT) acc[e] = 0.f;
        }
        float S[kRPT][16];
#pragma unroll
        for (int rr = 0; rr < kRPT; ++rr)
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 s4 = *reinterpret_cast<const float4 *>(ck_raw + stage * kN * kN +
                                                                    (row0 + rr) * kN + 16 * m + 4 * q);
                S[rr][4 * m] = s4.x; S[rr][4 * m + 1] = s4.y; S[rr][4 * m + 2] = s4.z; S[rr][4 * m + 3] = s4.w;
            }
        __syncthreads();
        if (c > 0) issue_chunk(c - 1, stage ^ 1);

        auto vec = [&](int ten, int tt) { return fbuf + (ten * CK + tt) * kN; };

        // ---- recompute the chunk's states ------------------------------------
        for (int tt = 0; tt < L; ++tt) {
#pragma unroll
            for (int rr = 0; rr < kRPT; ++rr)
#pragma unroll
                for (int m = 0; m < 4; ++m)
                    __stcg(&my_hist[((size_t)tt * (kRPT * 4) + rr * 4 + m) * kNT + tid],
                           make_float4(S[rr][4 * m], S[rr][4 * m + 1], S[rr][4 * m + 2], S[rr][4 * m + 3]));
            const float *av = vec(4, tt), *wv = vec(1, tt), *bv = vec(5, tt), *kv = vec(2, tt), *vv = vec(3, tt);
            float p[kRPT] = {};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 a4 = *reinterpret_cast<const float4 *>(av + 16 * m + 4 * q);
#pragma unroll
                for (int rr = 0; rr < kRPT; ++rr) {
                    p[rr] = fmaf(S[rr][4 * m + 0], a4.x, p[rr]);
                    p[rr] = fmaf(S[rr][4 * m + 1], a4.y, p[rr]);
                    p[rr] = fmaf(S[rr][4 * m + 2], a4.z, p[rr]);
                    p[rr] = fmaf(S[rr][4 * m + 3], a4.w, p[rr]);
                }
            }
#pragma unroll
            for (int rr = 0; rr < kRPT; ++rr) {
                p[rr] += __shfl_xor_sync(0xffffffffu, p[rr], 1);
                p[rr] += __shfl_xor_sync(0xffffffffu, p[rr], 2);
                if (q == rr) p_s[tt * kN + row0 + rr] = p[rr];
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 w4 = *reinterpret_cast<const float4 *>(wv + 16 * m + 4 * q);
                const float4 b4 = *reinterpret_cast<const float4 *>(bv + 16 * m + 4 * q);
                const float4 k4 = *reinterpret_cast<const float4 *>(kv + 16 * m + 4 * q);
                const float wj[4] = {w4.x, w4.y, w4.z, w4.w};
                const float bj[4] = {b4.x, b4.y, b4.z, b4.w};
                const float kj[4] = {k4.x, k4.y, k4.z, k4.w};
#pragma unroll
                for (int rr = 0; rr < kRPT; ++rr) {
                    const float vi = vv[row0 + rr];
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        S[rr][4 * m + e] = fmaf(S[rr][4 * m + e], wj[e], fmaf(p[rr], bj[e], vi * kj[e]));
                }
            }
        }
        __syncwarp();
        __syncthreads();   // p_s visible to all lanes

        // ---- reverse sweep -----------------------------------------------------
        for (int tt = L - 1; tt >= 0; --tt) {
            const float *rv = vec(0, tt), *wv = vec(1, tt), *kv = vec(2, tt), *vv = vec(3, tt);
            const float *av = vec(4, tt), *bv = vec(5, tt), *dyv = vec(6, tt);
            float Sp[kRPT][16];
#pragma unroll
            for (int rr = 0; rr < kRPT; ++rr)
#pragma unroll
                for (int m = 0; m < 4; ++m) {
                    const float4 s4 = __ldcg(&my_hist[((size_t)tt * (kRPT * 4) + rr * 4 + m) * kNT + tid]);
                    Sp[rr][4 * m] = s4.x; Sp[rr][4 * m + 1] = s4.y; Sp[rr][4 * m + 2] = s4.z; Sp[rr][4 * m + 3] = s4.w;
                }
            float dyi[kRPT], vi[kRPT], pi[kRPT];
#pragma unroll
            for (int rr = 0; rr < kRPT; ++rr) {
                dyi[rr] = dyv[row0 + rr];
                vi[rr] = vv[row0 + rr];
                pi[rr] = p_s[tt * kN + row0 + rr];
            }
            // vals: [0,16) dr  [16,32) dk  [32,48) dw  [48,64) db  [64,80) da
            float vals[80];
            float dvp[kRPT] = {}, dpp[kRPT] = {};
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 r4 = *reinterpret_cast<const float4 *>(rv + 16 * m + 4 * q);
                const float4 k4 = *reinterpret_cast<const float4 *>(kv + 16 * m + 4 * q);
                const float4 b4 = *reinterpret_cast<const float4 *>(bv + 16 * m + 4 * q);
                const float rj[4] = {r4.x, r4.y, r4.z, r4.w};
                const float kj[4] = {k4.x, k4.y, k4.z, k4.w};
                const float bj[4] = {b4.x, b4.y, b4.z, b4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 4 * m + e;
                    float drs = 0.f, dks = 0.f, dws = 0.f, dbs = 0.f;
#pragma unroll
                    for (int rr = 0; rr < kRPT; ++rr) {
                        drs = fmaf(dyi[rr], S[rr][c], drs);
                        const float gg = fmaf(dyi[rr], rj[e], g[rr][c]);
                        g[rr][c] = gg;
                        dvp[rr] = fmaf(gg, kj[e], dvp[rr]);
                        dpp[rr] = fmaf(gg, bj[e], dpp[rr]);
                        dks = fmaf(vi[rr], gg, dks);
                        dws = fmaf(Sp[rr][c], gg, dws);
                        dbs = fmaf(pi[rr], gg, dbs);
                    }
                    vals[c] = drs;
                    vals[16 + c] = dks;
                    vals[32 + c] = dws;
                    vals[48 + c] = dbs;
                }
            }
#pragma unroll
            for (int rr = 0; rr < kRPT; ++rr) {
                dvp[rr] += __shfl_xor_sync(0xffffffffu, dvp[rr], 1);
                dvp[rr] += __shfl_xor_sync(0xffffffffu, dvp[rr], 2);
                dpp[rr] += __shfl_xor_sync(0xffffffffu, dpp[rr], 1);
                dpp[rr] += __shfl_xor_sync(0xffffffffu, dpp[rr], 2);
                if (q == rr) dv[base + (size_t)(t0 + tt) * tok_stride + row0 + rr] = from_f32<GradT>(dvp[rr]);
            }
#pragma unroll
            for (int m = 0; m < 4; ++m) {
                const float4 w4 = *reinterpret_cast<const float4 *>(wv + 16 * m + 4 * q);
                const float4 a4 = *reinterpret_cast<const float4 *>(av + 16 * m + 4 * q);
                const float wj[4] = {w4.x, w4.y, w4.z, w4.w};
                const float aj[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int c = 4 * m + e;
                    float das = 0.f;
#pragma unroll
                    for (int rr = 0; rr < kRPT; ++rr) {
                        das = fmaf(dpp[rr], Sp[rr][c], das);
                        g[rr][c] = fmaf(g[rr][c], wj[e], dpp[rr] * aj[e]);
                        S[rr][c] = Sp[rr][c];
                    }
                    vals[64 + c] = das;
                }
            }
            // reduce the 80 column partials over the warp's 8 row groups
            rs_step<80>(vals, 16);
            rs_step<40>(vals, 8);
            rs_step<20>(vals, 4);
            const int lane = tid & 31;
            const int first = ((lane >> 4) & 1) * 40 + ((lane >> 3) & 1) * 20 + ((lane >> 2) & 1) * 10;
            float *acc_t = acc + tt * kNRED * kN;
#pragma unroll
            for (int i = 0; i < 10; ++i) {
                const int idx = first + i;          // = vector * 16 + c
                const int vecid = idx >> 4, cc = idx & 15;
                const int j = 16 * (cc >> 2) + 4 * q + (cc & 3);
                atomicAdd(acc_t + vecid * kN + j, vals[i]);
            }
        }
        __syncthreads();
        // ---- write the chunk's row-summed gradients ------------------------------
        GradT *outs[kNRED] = {dr, dk, dw, db, da};
        for (int e = tid * 4; e < L * kNRED * kN; e += kNT * 4) {
            const int tt = e / (kNRED * kN);
            const int rem = e % (kNRED * kN);
            const int vecid = rem / kN, j = rem % kN;
            store4(outs[vecid] + base + (size_t)(t0 + tt) * tok_stride + j,
                   *reinterpret_cast<const float4 *>(acc + e));
        }
    }

#pragma unroll
    for (int rr = 0; rr < kRPT; ++rr)
#pragma unroll
        for (int m = 0; m < 4; ++m)
            store4(ds0 + st_base + (size_t)(row0 + rr) * kN + 16 * m + 4 * q,
                   make_float4(g[rr][4 * m], g[rr][4 * m + 1], g[rr][4 * m + 2], g[rr][4 * m + 3]));
}

size_t bwd_smem_bytes(int CK, wkv7_dtype in_dt) {
    const size_t es = in_dt == WKV7_F32 ? 4 : 2;
    return 2 * kNTEN * CK * kN * es + 2 * kN * kN * 4 + (size_t)kNTEN * CK * kN * 4 +
           (size_t)CK * kNRED * kN * 4 + (size_t)CK * kN * 4;
}

size_t bwd_hist_bytes(int B, int H, int CK) { return (size_t)B * H * CK * kN * kN * sizeof(float); }

cudaError_t bwd_seq(int B, int T, int H, int CK, wkv7_dtype in_dt, wkv7_dtype g_dt, const void *r,
                    const void *w, const void *k, const void *v, const void *a, const void *b,
                    const void *dy, const float *dsT, const float *ckpt, float *hist, void *dr, void *dw,
                    void *dk, void *dv, void *da, void *db, float *ds0, cudaStream_t st) {
    const size_t smem = bwd_smem_bytes(CK, in_dt);
#define WKV7_BWD_LAUNCH(I, G)                                                                          \
    do {                                                                                                \
        auto kern = bwd_seq_kernel<I, G>;                                                               \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem); \
        if (e != cudaSuccess) return e;                                                                 \
        kern<<<B * H, kNT, smem, st>>>(T, H, CK, (const I *)r, (const I *)w, (const I *)k, (const I *)v,  \
                                       (const I *)a, (const I *)b, (const I *)dy, dsT, ckpt,            \
                                       reinterpret_cast<float4 *>(hist), (G *)dr, (G *)dw, (G *)dk,     \
                                       (G *)dv, (G *)da, (G *)db, ds0);                                 \
    } while (0)
    if (in_dt == WKV7_F32 && g_dt == WKV7_F32) WKV7_BWD_LAUNCH(float, float);
    else if (in_dt == WKV7_F32) WKV7_BWD_LAUNCH(float, __nv_bfloat16);
    else if (g_dt == WKV7_F32) WKV7_BWD_LAUNCH(__nv_bfloat16, float);
    else WKV7_BWD_LAUNCH(__nv_bfloat16, __nv_bfloat16);
#undef WKV7_BWD_LAUNCH
    return cudaGetLastError();
}

}  // namespace wkv7
