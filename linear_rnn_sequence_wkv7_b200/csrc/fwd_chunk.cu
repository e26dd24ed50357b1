// Chunked WKV7 forward on the sm_100a tensor cores (tcgen05, TMEM accumulators).
//
// The pages state that RWKV-7 keeps training parallelisable (RWKV-7 "Goose"
// with Expressive Dynamic State Evolution, abstract) and cite chunk-wise
// parallelisation of the delta rule only by title; the algebra below is our
// own derivation from the recurrence
//     S_t = S_{t-1} (diag(w_t) + a_t b_t^T) + v_t k_t^T,   y_t = S_t r_t.
//
// Chunk of L = 32 tokens (local t, s in [0, 32)), entry state S (64 x 64,
// row i = value, column j = key).  Per channel, with the suffix products
// p_t = prod_{m >= t} w_m and G = p_0 (the chunk's total decay):
//   a'_t = a_t / p_t,   r'_t = r_t / p_{t+1},   b-_t = b_t p_{t+1},
//   k-_t = k_t p_{t+1}                                (p_32 = 1)
// so that a'_t . b-_s = sum_j a_t b_s prod_{s<m<t} w_m, the decayed
// interaction of token t's removal read with token s's write, etc.
//   Gram  = [a'; r'] [b-; k-]^T                        (64 x 64)
//   L_ab, L_ak = strictly lower parts of the a' rows; L_rb, L_rk = lower
//                parts of the r' rows (diagonal included)
//   W' = (I - L_ab)^{-1} A',  U~ = (I - L_ab)^{-1} L_ak V
//            (fp32 forward substitution on the CUDA cores; u_t = S G w'_t + u~_t)
//   M = G (I + W'^T B-),  Q^T = G (R'^T + W'^T L_rb^T)   (G scales rows)
//   E = U~^T B- + V^T K-,  Y_loc^T = U~^T L_rb^T + V^T L_rk^T
//   S_out = S M + E,  Y^T = S Q^T + Y_loc^T          (state-dependent part)
//
// Precision: every tensor-core product uses bf16 hi/lo splits (x = hi + lo to
// 16 bits; three passes hi*hi + hi*lo + lo*hi, two when one side is an exact
// bf16 input such as v) with fp32 accumulation in TMEM.  A single tf32 or bf16
// pass is not accurate enough for the 2e-3 rms bound on this workload.
//
// Mapping: one CTA (256 threads, 8 warps) per (b, h), two CTAs per SM;
// chunks are processed in order.  Per chunk: P0 builds the decayed operands
// from the token tile (suffix products by warp shuffles); R1 Gram; P1 masks
// it; P1b solves W' and U~ by forward substitution; R3 M'', Q''^T, E,
// Y_loc^T; P3 finishes M and Q; R4 accumulates the state product onto
// [E | Y_loc^T]; P4 writes y and stages S_out as the next chunk's operand.
// The rounds are software-pipelined across chunks: R4 of chunk c runs under
// P0 of chunk c+1, and R1 of chunk c+1 under P4 of chunk c.  One thread issues
// the MMAs; completion is tracked by an mbarrier with a bounded wait.  Token
// tiles are fetched with cp.async two chunks ahead of use.
//
// TMEM (256 columns; an M=64 accumulator occupies lanes 16q..16q+15 of warp
// quadrant q):
//   X: cols [0, 96)    Gram (64), then M'' (64) | Q''^T (32)
//   Z: cols [128, 224) [E | Y_loc^T], then += S [M | Q^T]
#include "umma.cuh"

namespace wkv7 {

namespace chunk {

constexpr int L = 32;          // tokens per chunk
constexpr int NT = 256;        // threads per CTA
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_X = 0, COL_Z = 128;

// shared memory map (bytes)
constexpr uint32_t IN = 0;     // token tile: tensors w r k a b v, [32][128 B] each, 16-B chunks rotated by row
constexpr uint32_t IN_W = 0, IN_R = 4096, IN_K = 8192, IN_A = 12288, IN_B = 16384, IN_V = 20480;
constexpr uint32_t GA_HI = 24576, GA_LO = 32768;     // [64][64]: a' rows 0..31, r' rows 32..63
constexpr uint32_t GBK_HI = 40960, GBK_LO = 49152;   // [64][64]: b- rows 0..31, k- rows 32..63
constexpr uint32_t VB = 57344;                       // [32][64] exact bf16 v
constexpr uint32_t LRB_HI = 61440, LRB_LO = 63488, LRK_HI = 65536, LRK_LO = 67584;   // [32][32]
constexpr uint32_t S_HI = 69632, S_LO = 77824;       // [64][64]
constexpr uint32_t SCR = 86016;                      // 24 KB with three successive lives:
constexpr uint32_t LABT = SCR, LAKT = SCR + 4096;    //  P1..P1b: fp32 [32][32] L_ab^T, L_ak^T
constexpr uint32_t WT_HI = SCR + 8192, WT_LO = SCR + 12288, UT_HI = SCR + 16384, UT_LO = SCR + 20480;  // [64][32]
constexpr uint32_t M_HI = SCR, M_LO = SCR + 8192, Q_HI = SCR + 16384, Q_LO = SCR + 20480;  //  P3..R4
constexpr uint32_t YSM = SCR;                        //  P4: fp32 [32][64] y tile
constexpr uint32_t GAML = 110592;                    // fp32 [64]: G per channel
constexpr uint32_t MBAR = 110848;                    // u64
constexpr uint32_t TMEM_SLOT = 110856;               // u32
constexpr uint32_t FLAG = 110860;                    // u32 abort flag
constexpr uint32_t SMEM_BYTES = 110864;

constexpr long long kWaitCycles = 2000000000LL;      // ~1 s: far above any legitimate MMA round
constexpr float kMinDecay = 1e-30f;                  // per-chunk decay floor (prod of 32 w)

__device__ __forceinline__ uint32_t in_off(int t, int ch) { return (uint32_t)(t * 128 + (((ch + t) & 7) << 4)); }

__device__ __forceinline__ void bf8_to_f32(uint4 u, float *o) {
    const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        o[2 * q] = __uint_as_float(uu[q] << 16);
        o[2 * q + 1] = __uint_as_float(uu[q] & 0xffff0000u);
    }
}

__device__ __forceinline__ float bf_at(const unsigned char *p) {
    return __uint_as_float((uint32_t)(*reinterpret_cast<const unsigned short *>(p)) << 16);
}

}  // namespace chunk

template <typename OutT>
__global__ void __launch_bounds__(chunk::NT, 2)
fwd_chunk_kernel(int T, int H, const __nv_bfloat16 *__restrict__ r, const __nv_bfloat16 *__restrict__ w,
                 const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
                 const __nv_bfloat16 *__restrict__ a, const __nv_bfloat16 *__restrict__ b,
                 const float *s0, OutT *__restrict__ y, float *sT) {
    using namespace chunk;
    using namespace umma;
    extern __shared__ __align__(1024) unsigned char sm[];
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int q4 = warp & 3, hc = warp >> 2;             // TMEM lane quadrant, column half
    const int h = blockIdx.x, bb = blockIdx.y;
    const size_t tok_stride = (size_t)H * kN;
    const size_t base = ((size_t)bb * T * H + h) * kN;
    const size_t st_base = ((size_t)bb * H + h) * kN * kN;
    const int nchunks = (T + L - 1) / L;
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(sm + FLAG);
    const uint32_t mbar = sbase + MBAR;

    auto issue_tile = [&](int c) {
        const __nv_bfloat16 *src[6] = {w, r, k, a, b, v};
        const int t0 = c * L;
        for (int x = tid; x < 6 * L * 8; x += NT) {
            const int ten = x >> 8, t = (x >> 3) & 31, ch = x & 7;
            if (t0 + t < T)
                cp_async16(sm + IN + ten * 4096 + in_off(t, ch), src[ten] + base + (size_t)(t0 + t) * tok_stride + ch * 8);
        }
        cp_async_commit();
    };

    // ---- set-up -------------------------------------------------------------------------
    if (tid == 0) {
        mbar_init(mbar, 1);
        *abort_flag = 0;
    }
    if (warp == 0) tmem_alloc(sbase + TMEM_SLOT, TMEM_COLS);
    issue_tile(0);
    {
        const int i = tid >> 2, c0 = (tid & 3) * 16;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            float x[8];
            if (s0) {
                const float4 u0 = load4(s0 + st_base + (size_t)i * kN + c0 + 8 * g);
                const float4 u1 = load4(s0 + st_base + (size_t)i * kN + c0 + 8 * g + 4);
                x[0] = u0.x; x[1] = u0.y; x[2] = u0.z; x[3] = u0.w; x[4] = u1.x; x[5] = u1.y; x[6] = u1.z; x[7] = u1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = 0.f;
            }
            store8_split(sm + S_HI, sm + S_LO, cm_off(i, c0 + 8 * g, 64), x);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + TMEM_SLOT);
    const uint32_t quad = (uint32_t)(32 * q4) << 16;
    uint32_t phase = 0;

    auto round_wait = [&]() -> bool {
        const bool ok = mbar_wait(mbar, phase, kWaitCycles);
        phase ^= 1u;
        if (!ok) *abort_flag = 1;
        __syncthreads();
        fence_after_sync();
        return *abort_flag == 0;
    };
    auto issue_begin = [&]() {
        fence_smem_to_async();
        fence_before_sync();
        __syncthreads();
    };

    // ---- phases -------------------------------------------------------------------------
    auto P0 = [&](int Lv) {                       // decayed operands of one chunk
        const int g = warp, t = lane;             // channels 8g..8g+7, token t
        const bool valid = t < Lv;
        const uint32_t off = in_off(t, g);
        float wv[8], rv[8], kv[8], av[8], bv[8];
        bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + IN_W + off), wv);
        bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + IN_R + off), rv);
        bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + IN_K + off), kv);
        bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + IN_A + off), av);
        bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + IN_B + off), bv);
        const uint4 vraw = valid ? *reinterpret_cast<const uint4 *>(sm + IN_V + off) : make_uint4(0, 0, 0, 0);
        float inc[8], nxt[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            if (!valid) { wv[e] = 1.f; rv[e] = 0.f; kv[e] = 0.f; av[e] = 0.f; bv[e] = 0.f; }
            inc[e] = wv[e];
        }
#pragma unroll
        for (int o = 1; o < 32; o <<= 1)
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float up = __shfl_down_sync(0xffffffffu, inc[e], o);
                if (lane + o < 32) inc[e] *= up;
            }
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            const float n1 = __shfl_down_sync(0xffffffffu, inc[e], 1);
            nxt[e] = lane == 31 ? 1.f : n1;
            const float G = __shfl_sync(0xffffffffu, inc[e], 0);
            if (lane == 0) {
                reinterpret_cast<float *>(sm + GAML)[8 * g + e] = G;
                if (G < kMinDecay) raise_status(WKV7_ERR_RANGE);
            }
        }
        float xa[8], xr[8], xb[8], xk[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
            xa[e] = __fdividef(av[e], inc[e]);
            xr[e] = __fdividef(rv[e], nxt[e]);
            xb[e] = bv[e] * nxt[e];
            xk[e] = kv[e] * nxt[e];
        }
        store8_split(sm + GA_HI, sm + GA_LO, cm_off(t, 8 * g, 64), xa);
        store8_split(sm + GA_HI, sm + GA_LO, cm_off(L + t, 8 * g, 64), xr);
        store8_split(sm + GBK_HI, sm + GBK_LO, cm_off(t, 8 * g, 64), xb);
        store8_split(sm + GBK_HI, sm + GBK_LO, cm_off(L + t, 8 * g, 64), xk);
        *reinterpret_cast<uint4 *>(sm + VB + cm_off(t, 8 * g, 64)) = vraw;
    };

    auto issue_R1 = [&]() {
        fence_after_sync();
        gemm_split_d(tmem + COL_X, opd_k(sbase + GA_HI, sbase + GA_LO, 64), opd_k(sbase + GBK_HI, sbase + GBK_LO, 64),
                     idesc_bf16(64, 64, 0, 0), 4, false);
        commit(mbar);
    };

    auto P1 = [&]() {                             // mask the Gram into L_ab^T, L_ak^T (fp32), L_rb, L_rk (split)
        uint32_t r0[16], r1[16];
        tmem_ld16_nowait(tmem + quad + COL_X + 32 * hc, r0);
        tmem_ld16_nowait(tmem + quad + COL_X + 32 * hc + 16, r1);
        tmem_wait();
        if (lane < 16) {
            const int rho = 16 * q4 + lane;
            float g[32];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                g[e] = __uint_as_float(r0[e]);
                g[16 + e] = __uint_as_float(r1[e]);
            }
            if (rho < L) {
                const int t = rho;
                float *dst = reinterpret_cast<float *>(sm + (hc == 0 ? LABT : LAKT));
#pragma unroll
                for (int s = 0; s < L; ++s) dst[s * L + t] = s < t ? g[s] : 0.f;
            } else {
                const int t = rho - L;
                unsigned char *hi = sm + (hc == 0 ? LRB_HI : LRK_HI);
                unsigned char *lo = sm + (hc == 0 ? LRB_LO : LRK_LO);
#pragma unroll
                for (int qq = 0; qq < 4; ++qq) {
                    float x[8];
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = (8 * qq + e <= t) ? g[8 * qq + e] : 0.f;
                    store8_split(hi, lo, cm_off(t, 8 * qq, L), x);
                }
            }
        }
    };

    auto P1b = [&]() {                            // forward substitution for W' and U~ (column per thread)
        if (tid < 2 * kN) {
            const bool is_w = tid < kN;
            const int col = tid & 63;
            const float *labt = reinterpret_cast<const float *>(sm + LABT);
            const float *lakt = reinterpret_cast<const float *>(sm + LAKT);
            float acc[L];
#pragma unroll
            for (int t = 0; t < L; ++t) {
                const uint32_t o = cm_off(t, col, 64);
                acc[t] = is_w ? bf_at(sm + GA_HI + o) + bf_at(sm + GA_LO + o) : 0.f;
            }
#pragma unroll
            for (int m = 0; m < L; ++m) {
                const float x = acc[m];
                const float vm = is_w ? 0.f : bf_at(sm + VB + cm_off(m, col, 64));
#pragma unroll
                for (int c4 = (m + 1) / 4; c4 < L / 4; ++c4) {
                    const float4 lab = *reinterpret_cast<const float4 *>(labt + m * L + 4 * c4);
                    const float4 lak = *reinterpret_cast<const float4 *>(lakt + m * L + 4 * c4);
                    const float la[4] = {lab.x, lab.y, lab.z, lab.w};
                    const float lk[4] = {lak.x, lak.y, lak.z, lak.w};
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const int t = 4 * c4 + e;
                        if (t > m) acc[t] = fmaf(la[e], x, fmaf(lk[e], vm, acc[t]));
                    }
                }
            }
            unsigned char *hi = sm + (is_w ? WT_HI : UT_HI);
            unsigned char *lo = sm + (is_w ? WT_LO : UT_LO);
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) store8_split(hi, lo, cm_off(col, 8 * qq, L), acc + 8 * qq);
        }
    };

    auto issue_R3 = [&]() {
        fence_after_sync();
        const OpD wt = opd_k(sbase + WT_HI, sbase + WT_LO, L);
        const OpD ut = opd_k(sbase + UT_HI, sbase + UT_LO, L);
        const OpD vt = opd_mn(sbase + VB, 0, 64);
        const OpD bbar = opd_mn(sbase + GBK_HI, sbase + GBK_LO, 64);
        const OpD kbar = opd_mn(sbase + GBK_HI + 4096, sbase + GBK_LO + 4096, 64);
        const OpD lrb = opd_k(sbase + LRB_HI, sbase + LRB_LO, L);
        const OpD lrk = opd_k(sbase + LRK_HI, sbase + LRK_LO, L);
        gemm_split_d(tmem + COL_X, wt, bbar, idesc_bf16(64, 64, 0, 1), 2, false);
        gemm_split_d(tmem + COL_X + 64, wt, lrb, idesc_bf16(64, 32, 0, 0), 2, false);
        gemm_split_d(tmem + COL_Z, ut, bbar, idesc_bf16(64, 64, 0, 1), 2, false);
        gemm_split_d(tmem + COL_Z, vt, kbar, idesc_bf16(64, 64, 1, 1), 2, true);
        gemm_split_d(tmem + COL_Z + 64, ut, lrb, idesc_bf16(64, 32, 0, 0), 2, false);
        gemm_split_d(tmem + COL_Z + 64, vt, lrk, idesc_bf16(64, 32, 1, 0), 2, true);
        commit(mbar);
    };

    auto P3 = [&]() {                             // M = G (I + M''), Q^T = G (R'^T + Q''^T)
        uint32_t r0[16], r1[16], r2[16];
        tmem_ld16_nowait(tmem + quad + COL_X + 32 * hc, r0);
        tmem_ld16_nowait(tmem + quad + COL_X + 32 * hc + 16, r1);
        tmem_ld16_nowait(tmem + quad + COL_X + 64 + 16 * hc, r2);
        tmem_wait();
        if (lane < 16) {
            const int j = 16 * q4 + lane;
            const float G = reinterpret_cast<const float *>(sm + GAML)[j];
            float m[32];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                m[e] = G * (__uint_as_float(r0[e]) + (32 * hc + e == j ? 1.f : 0.f));
                m[16 + e] = G * (__uint_as_float(r1[e]) + (32 * hc + 16 + e == j ? 1.f : 0.f));
            }
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) store8_split(sm + M_HI, sm + M_LO, cm_off(j, 32 * hc + 8 * qq, 64), m + 8 * qq);
            float qv[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                const uint32_t o = cm_off(L + 16 * hc + e, j, 64);
                qv[e] = G * (__uint_as_float(r2[e]) + bf_at(sm + GA_HI + o) + bf_at(sm + GA_LO + o));
            }
#pragma unroll
            for (int qq = 0; qq < 2; ++qq) store8_split(sm + Q_HI, sm + Q_LO, cm_off(j, 16 * hc + 8 * qq, L), qv + 8 * qq);
        }
    };

    auto issue_R4 = [&]() {
        fence_after_sync();
        const OpD s = opd_k(sbase + S_HI, sbase + S_LO, 64);
        gemm_split_d(tmem + COL_Z, s, opd_mn(sbase + M_HI, sbase + M_LO, 64), idesc_bf16(64, 64, 0, 1), 4, true);
        gemm_split_d(tmem + COL_Z + 64, s, opd_mn(sbase + Q_HI, sbase + Q_LO, L), idesc_bf16(64, 32, 0, 1), 4, true);
        commit(mbar);
    };

    auto P4 = [&](int c, int Lv) {                // y, next S operand, final state
        uint32_t r0[16], r1[16], r2[16];
        tmem_ld16_nowait(tmem + quad + COL_Z + 32 * hc, r0);
        tmem_ld16_nowait(tmem + quad + COL_Z + 32 * hc + 16, r1);
        tmem_ld16_nowait(tmem + quad + COL_Z + 64 + 16 * hc, r2);
        tmem_wait();
        if (lane < 16) {
            const int i = 16 * q4 + lane;
            float sv[32];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                sv[e] = __uint_as_float(r0[e]);
                sv[16 + e] = __uint_as_float(r1[e]);
            }
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) store8_split(sm + S_HI, sm + S_LO, cm_off(i, 32 * hc + 8 * qq, 64), sv + 8 * qq);
            if (c == nchunks - 1 && sT) {
#pragma unroll
                for (int qq = 0; qq < 8; ++qq)
                    store4(sT + st_base + (size_t)i * kN + 32 * hc + 4 * qq,
                           make_float4(sv[4 * qq], sv[4 * qq + 1], sv[4 * qq + 2], sv[4 * qq + 3]));
            }
            float *ysm = reinterpret_cast<float *>(sm + YSM);
#pragma unroll
            for (int e = 0; e < 16; ++e) ysm[(16 * hc + e) * kN + i] = __uint_as_float(r2[e]);
        }
        fence_smem_to_async();
        fence_before_sync();
        __syncthreads();
        {   // coalesced y rows: thread -> (token, 8 channels)
            const int t = tid >> 3, c8 = tid & 7;
            if (t < Lv) {
                const float *ysm = reinterpret_cast<const float *>(sm + YSM) + t * kN + 8 * c8;
                OutT *dst = y + base + (size_t)(c * L + t) * tok_stride + 8 * c8;
                store4(dst, *reinterpret_cast<const float4 *>(ysm));
                store4(dst + 4, *reinterpret_cast<const float4 *>(ysm + 4));
            }
        }
        __syncthreads();
    };

    // ---- software-pipelined chunk loop ----------------------------------------------------
    auto run = [&]() {
        cp_async_wait<0>();
        __syncthreads();
        P0(min(L, T));
        __syncthreads();
        if (nchunks > 1) issue_tile(1);
        issue_begin();
        if (tid == 0) issue_R1();
        if (!round_wait()) return;
        P1();
        __syncthreads();
        P1b();
        issue_begin();
        if (tid == 0) issue_R3();
        if (!round_wait()) return;
        P3();
        issue_begin();
        if (tid == 0) issue_R4();
        for (int c = 0; c < nchunks; ++c) {
            const bool has_next = c + 1 < nchunks;
            if (has_next) {
                cp_async_wait<0>();
                __syncthreads();
                P0(min(L, T - (c + 1) * L));
                __syncthreads();
                if (c + 2 < nchunks) issue_tile(c + 2);
            }
            if (!round_wait()) return;                       // R4(c)
            if (has_next) {
                issue_begin();
                if (tid == 0) issue_R1();                    // R1(c+1), overlapped with P4(c)
            }
            P4(c, min(L, T - c * L));
            if (has_next) {
                if (!round_wait()) return;                   // R1(c+1)
                P1();
                __syncthreads();
                P1b();
                issue_begin();
                if (tid == 0) issue_R3();
                if (!round_wait()) return;
                P3();
                issue_begin();
                if (tid == 0) issue_R4();                    // R4(c+1), overlapped with P0(c+2)
            }
        }
    };
    run();

    // ---- tear-down ----------------------------------------------------------------------
    cp_async_wait<0>();
    __syncthreads();
    if (*abort_flag) {
        // a tensor-core round did not complete in time: report it, give the
        // in-flight work one more bounded wait, then release TMEM
        if (tid == 0) raise_status(WKV7_ERR_TIMEOUT);
        mbar_wait(mbar, phase ^ 1u, kWaitCycles);
        __syncthreads();
    }
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

cudaError_t fwd_chunk(int B, int T, int H, wkv7_dtype y_dt, const void *r, const void *w, const void *k,
                      const void *v, const void *a, const void *b, const float *s0, void *y, float *sT,
                      cudaStream_t st) {
    dim3 grid(H, B);
    const size_t smem = chunk::SMEM_BYTES;
#define WKV7_CHUNK_LAUNCH(O)                                                                                 \
    do {                                                                                                     \
        auto kern = fwd_chunk_kernel<O>;                                                                     \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);  \
        if (e != cudaSuccess) return e;                                                                      \
        kern<<<grid, chunk::NT, smem, st>>>(T, H, (const __nv_bfloat16 *)r, (const __nv_bfloat16 *)w,        \
                                            (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,              \
                                            (const __nv_bfloat16 *)a, (const __nv_bfloat16 *)b, s0, (O *)y, sT); \
    } while (0)
    if (y_dt == WKV7_F32) WKV7_CHUNK_LAUNCH(float);
    else WKV7_CHUNK_LAUNCH(__nv_bfloat16);
#undef WKV7_CHUNK_LAUNCH
    return cudaGetLastError();
}

}  // namespace wkv7
