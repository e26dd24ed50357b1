// Chunked WKV7 backward.
//
// Gradient of L = sum(dy * y) + sum(dsT * sT) for the recurrence
//     S_t = S_{t-1} (diag(w_t) + a_t b_t^T) + v_t k_t^T,   y_t = S_t r_t
// (RWKV-7 "Goose" with Expressive Dynamic State Evolution: the generalised
// delta rule with vector decay; the pages give no backward, this is our own
// reverse-mode derivation of the chunked form).
//
// Three launches:
//  1. state checkpoints S_in(c) before every chunk of L = 32 tokens and the
//     final state (the chunked forward's epilogue for bf16 inputs,
//     fwd_chunk.cu; the sequential forward in checkpoint mode for fp32
//     inputs, fwd_seq.cu);
//  2. bwd_dstate_kernel: dS_out(c) = dL/dS at the end of every chunk, through
//     the chunk's own outputs excluded, by a reverse sweep of the state
//     gradient alone (per row i: g += dy_t[i] r_t; g = g w_t + (g . b_t) a_t);
//     it needs no state and no column sums (rows are independent, two CTAs
//     per head), and ends with ds0;
//  3. the chunks' input gradients, all chunks independent given S_in(c) and
//     dS_out(c): on the tensor cores for bf16 inputs (bwd_chunk_tc.cu), else
//     bwd_chunk_kernel below, one CTA per chunk with fp32 matrix products in
//     shared memory.
//
// Per chunk (local t, s in [0, L), suffix decay products p_t = prod_{m>=t} w_m,
// p_L = 1, G = p_0; all decay ratios that appear are <= 1):
//   a'_t = a_t / p_t,  r'_t = r_t / p_{t+1},  b-_s = b_s p_{s+1},  k-_s = k_s p_{s+1}
//   [L_ab L_ak; L_rb L_rk] = [a'; r'] [b-; k-]^T  (ab, ak strictly lower; rb, rk lower)
//   T = (I - L_ab)^{-1},  SG = S_in diag(G)
//   U   = T (a' SG^T + L_ak V)                        (rows u_t = S_{t-1} a_t)
//   dU  = b- dS^T + L_rb^T dY,   dZ = T^T dU
//   dV  = k- dS^T + L_rk^T dY + L_ak^T dZ
//   [dL_ab dL_ak; dL_rb dL_rk] = [dZ; dY] [U; V]^T  (same masks)
//   da = (dZ SG + dL_ab b- + dL_ak k-) / p_t
//   dr = (dY SG + dL_rb b- + dL_rk k-) / p_{t+1}
//   db = (U dS + dL_ab^T a' + dL_rb^T r') p_{s+1}
//   dk = (V dS + dL_ak^T a' + dL_rk^T r') p_{s+1}
//   q_t = dr_t r_t - db_t b_t - dk_t k_t + da_{t+1} a_{t+1} (t+1 < L)
//         + [t = L-1] sum_i S_out[i,:] dS[i,:]
//   dw_m = (sum_{t>=m} q_t) / w_m
// with dS = dS_out(c).  (q_t is the derivative through the prefix decay
// gamma_t = prod_{m<=t} w_m times gamma_t; dw_m = sum_{t>=m} dL/dgamma_t
// gamma_t / w_m.)
#include "common.cuh"

namespace wkv7 {

namespace bwdc {

constexpr int L = 32;          // tokens per chunk (the checkpoint interval)
constexpr int NT = 256;        // threads of the gradient kernel
constexpr int LD = 68;         // row pitch (floats) of 64-wide fp32 tiles
constexpr int LDS = 36;        // row pitch of 32-wide fp32 tiles
constexpr float kMinDecay = 1e-30f;

}  // namespace bwdc

// ---------------------------------------------------------------------------
// dS_out(c) for every chunk and ds0: reverse sweep of the state gradient.
// The rows of dS evolve independently.  LPR lanes per row (64 / LPR columns
// each, in groups of 4 at a stride of 4 LPR) and RPT rows per thread: with
// four lanes, RPT = 4 covers a (b, h) with a CTA of 64 threads, RPT = 2 with
// 128 threads, and RPT = 1 splits it over two CTAs of 128 (rows 32 q ..
// 32 q + 31) for problems with too few heads to fill the GPU; eight lanes and
// RPT = 4 make 128-thread CTAs, more warps per head at the same instructions
// per row.  More rows per thread share the conversions and loads of r, w, a, b.  Token tiles of r w a b dy are
// prefetched by cp.async, 32 tokens ahead.
//
// A launch runs nz segments of t_seg tokens (segment seg0 + z, whole chunks;
// only the last one of the sequence is ragged), each for all heads.  The
// sweep is affine in G: over a segment, G_in = G_out M^T + F with M the
// segment's transition product and F its own part (G_out = 0).  So a long
// sweep with few heads splits into segments: a dual run carries G from 0
// with dy (-> F) and a second G from I without dy (-> M^T) through one pass;
// the entry adjoints are chained from those, and an output run per segment
// sweeps again from its true G_out, storing dS_out.  In a DUAL launch only
// the last segment (z = nz - 1) is an output run.
//   g_in   : G at the segment's end per z (stride g_in_zstride), NULL = 0
//   g_out  : G at the segment's start, for runs z < g_out_nz
//   m_out  : the dual runs' M^T
// ---------------------------------------------------------------------------
template <typename InT, int RPT, int LPR, bool DUAL>
__global__ void __launch_bounds__(128)
bwd_dstate_kernel(int T, int t_seg, int seg0, int nz, const InT *__restrict__ r, const InT *__restrict__ w,
                  const InT *__restrict__ a, const InT *__restrict__ b, const InT *__restrict__ dy, int H,
                  const float *__restrict__ g_in, long long g_in_zstride, float *__restrict__ dS_out,
                  float *__restrict__ g_out, long long g_out_zstride, int g_out_nz, float *__restrict__ m_out,
                  long long m_zstride) {
    constexpr int L = bwdc::L, NTEN = 5, VEC = 16 / sizeof(InT), CPV = kN / VEC;
    constexpr int NR = DUAL ? 2 * RPT : RPT;   // rows RPT.. carry the dual run's second G
    constexpr int CPL = kN / LPR, NG = CPL / 4;   // columns per lane, in groups of 4 (stride 4 LPR)
    extern __shared__ __align__(16) unsigned char dsmem[];
    auto tile = reinterpret_cast<InT(*)[NTEN][L][kN]>(dsmem);   // [2 stages]
    constexpr int SPLIT = RPT == 1 ? 2 : 1;         // CTAs per head
    constexpr int NTH = LPR * kN / (SPLIT * RPT);   // threads: LPR lanes per group of RPT rows
    static_assert(NTH <= 128 && (LPR == 4 || LPR == 8), "sweep CTA shape");
    const int tid = threadIdx.x, q = tid % LPR;
    const int per_z = gridDim.x / nz;
    const int z = blockIdx.x / per_z, head = (blockIdx.x % per_z) / SPLIT;
    const int row0 = (SPLIT == 2 ? 32 * (blockIdx.x % 2) : 0) + RPT * (tid / LPR);
    const int bb = head / H, h = head % H;
    const size_t tok_stride = (size_t)H * kN;
    const size_t base = ((size_t)bb * T * H + h) * kN;
    const int nck_total = (T + L - 1) / L;
    const int t_begin = (seg0 + z) * t_seg, t_end = min(T, t_begin + t_seg);
    const int c_begin = t_begin / L, c_last = (t_end + L - 1) / L - 1;
    const bool out_run = !DUAL || z == nz - 1;
    const size_t hoff = (size_t)head * kN * kN;
    const InT *src[NTEN] = {r, w, a, b, dy};
    auto col = [&](int m) { return 4 * LPR * m + 4 * q; };   // first of this lane's 4 columns in group m

    auto issue = [&](int c, int stage) {
        const int t0 = c * L, Lc = min(L, T - t0);
#pragma unroll
        for (int ten = 0; ten < NTEN; ++ten)
            for (int x = tid; x < L * CPV; x += NTH) {
                const int tt = x / CPV, ch = x % CPV;
                if (tt < Lc)
                    cp_async16(&tile[stage][ten][tt][ch * VEC], src[ten] + base + (size_t)(t0 + tt) * tok_stride + ch * VEC);
            }
        cp_async_commit();
    };

    float g[NR][CPL];
#pragma unroll
    for (int rr = 0; rr < NR; ++rr)
#pragma unroll
        for (int m = 0; m < NG; ++m) {
            float4 d4 = make_float4(0.f, 0.f, 0.f, 0.f);
            const int row = row0 + rr % RPT, c0 = col(m);
            if (rr >= RPT) {             // identity start of the product run
                d4.x = row == c0 ? 1.f : 0.f;
                d4.y = row == c0 + 1 ? 1.f : 0.f;
                d4.z = row == c0 + 2 ? 1.f : 0.f;
                d4.w = row == c0 + 3 ? 1.f : 0.f;
            } else if (out_run && g_in) {
                d4 = load4(g_in + z * g_in_zstride + hoff + (size_t)row * kN + c0);
            }
            g[rr][4 * m] = d4.x; g[rr][4 * m + 1] = d4.y; g[rr][4 * m + 2] = d4.z; g[rr][4 * m + 3] = d4.w;
        }
    if (t_begin < t_end) issue(c_last, 0);   // an empty segment passes G through
    for (int c = c_last; c >= c_begin; --c) {
        const int stage = (c_last - c) & 1;
        const int t0 = c * L, Lc = min(L, T - t0);
        cp_async_wait<0>();
        __syncthreads();
        if (c > c_begin) issue(c - 1, stage ^ 1);
        if (out_run && dS_out) {   // dL/dS after the chunk's last token, before its own output is added
            float *dst = dS_out + ((size_t)head * nck_total + c) * kN * kN + (size_t)row0 * kN;
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
                for (int m = 0; m < NG; ++m)
                    store4(dst + (size_t)rr * kN + col(m),
                           make_float4(g[rr][4 * m], g[rr][4 * m + 1], g[rr][4 * m + 2], g[rr][4 * m + 3]));
        }
        for (int tt = Lc - 1; tt >= 0; --tt) {
            const InT *rv = tile[stage][0][tt], *wv = tile[stage][1][tt], *av = tile[stage][2][tt];
            const InT *bv = tile[stage][3][tt];
            // packed fp32 pairs (fma.rn.f32x2): the same per-element arithmetic as
            // scalar fmaf, half the FP instructions of an issue-bound loop
            float2 dyi[RPT], dp4[NR][2];  // four partial sums per row (two pairs)
#pragma unroll
            for (int rr = 0; rr < RPT; ++rr) {
                const float d = to_f32(tile[stage][4][tt][row0 + rr]);
                dyi[rr] = make_float2(d, d);
            }
#pragma unroll
            for (int rr = 0; rr < NR; ++rr) dp4[rr][0] = dp4[rr][1] = make_float2(0.f, 0.f);
#pragma unroll
            for (int m = 0; m < NG; ++m) {
                const float4 r4 = load4(rv + col(m)), b4 = load4(bv + col(m));
                const float2 rj[2] = {make_float2(r4.x, r4.y), make_float2(r4.z, r4.w)};
                const float2 bj[2] = {make_float2(b4.x, b4.y), make_float2(b4.z, b4.w)};
#pragma unroll
                for (int rr = 0; rr < NR; ++rr)
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        float2 gg = make_float2(g[rr][4 * m + 2 * e], g[rr][4 * m + 2 * e + 1]);
                        if (rr < RPT) gg = __ffma2_rn(dyi[rr], rj[e], gg);
                        g[rr][4 * m + 2 * e] = gg.x;
                        g[rr][4 * m + 2 * e + 1] = gg.y;
                        dp4[rr][e] = __ffma2_rn(gg, bj[e], dp4[rr][e]);
                    }
            }
            float dp[NR];
#pragma unroll
            for (int rr = 0; rr < NR; ++rr) {
                dp[rr] = (dp4[rr][0].x + dp4[rr][0].y) + (dp4[rr][1].x + dp4[rr][1].y);
#pragma unroll
                for (int o = 1; o < LPR; o <<= 1) dp[rr] += __shfl_xor_sync(0xffffffffu, dp[rr], o);
            }
#pragma unroll
            for (int m = 0; m < NG; ++m) {
                const float4 w4 = load4(wv + col(m)), a4 = load4(av + col(m));
                const float2 wj[2] = {make_float2(w4.x, w4.y), make_float2(w4.z, w4.w)};
                const float2 aj[2] = {make_float2(a4.x, a4.y), make_float2(a4.z, a4.w)};
#pragma unroll
                for (int rr = 0; rr < NR; ++rr) {
                    const float2 dpp = make_float2(dp[rr], dp[rr]);
#pragma unroll
                    for (int e = 0; e < 2; ++e) {
                        const float2 gg = __ffma2_rn(make_float2(g[rr][4 * m + 2 * e], g[rr][4 * m + 2 * e + 1]),
                                                     wj[e], __fmul2_rn(dpp, aj[e]));
                        g[rr][4 * m + 2 * e] = gg.x;
                        g[rr][4 * m + 2 * e + 1] = gg.y;
                    }
                }
            }
        }
    }
    auto store_rows = [&](float *dst, int r_first) {
#pragma unroll
        for (int rr = 0; rr < RPT; ++rr)
#pragma unroll
            for (int m = 0; m < NG; ++m)
                store4(dst + hoff + (size_t)(row0 + rr) * kN + col(m),
                       make_float4(g[r_first + rr][4 * m], g[r_first + rr][4 * m + 1], g[r_first + rr][4 * m + 2],
                                   g[r_first + rr][4 * m + 3]));
    };
    if (z < g_out_nz) store_rows(g_out + z * g_out_zstride, 0);
    if (DUAL && !out_run) store_rows(m_out + z * m_zstride, DUAL ? RPT : 0);
}

// ---------------------------------------------------------------------------
// fp32 products in shared memory for the gradient kernel (256 threads).
// C is M x 64 (M = 64 or 32); thread tid owns rows m0 .. m0 + RM - 1
// (RM = 4 or 2, m0 = RM * (tid >> 4)) and columns n0 .. n0 + 3 (n0 = 4 (tid & 15)).
// B(k, n) is read row-major, B[k * ldb + n]; A(m, k) either row-major
// (A[m * lda + k]) or column-major (A[k * lda + m], vector loads).
// ---------------------------------------------------------------------------
namespace bwdc {

template <int M>
struct Acc {
    static constexpr int RM = M == 64 ? 4 : 2;
    float c[RM][4];
    __device__ __forceinline__ void zero() {
#pragma unroll
        for (int i = 0; i < RM; ++i)
#pragma unroll
            for (int j = 0; j < 4; ++j) c[i][j] = 0.f;
    }
};

template <int M, bool A_COL>
__device__ __forceinline__ void load_a(float (&av)[Acc<M>::RM], const float *A, int lda, int k, int m0) {
    constexpr int RM = Acc<M>::RM;
    if constexpr (A_COL) {
        if constexpr (RM == 4) {
            const float4 a4 = *reinterpret_cast<const float4 *>(A + (size_t)k * lda + m0);
            av[0] = a4.x; av[1] = a4.y; av[2] = a4.z; av[3] = a4.w;
        } else {
            const float2 a2 = *reinterpret_cast<const float2 *>(A + (size_t)k * lda + m0);
            av[0] = a2.x; av[1] = a2.y;
        }
    } else {
#pragma unroll
        for (int i = 0; i < RM; ++i) av[i] = A[(size_t)(m0 + i) * lda + k];
    }
}

// K is a multiple of 4.  A row-major (A[m * lda + k]): four k steps per pass,
// each thread's A rows read as float4 along k (one load per row and pass
// instead of one per row and k).  A column-major (A[k * lda + m]): the
// operands of step k + 1 are loaded while step k is multiplied.
template <int M, bool A_COL>
__device__ __forceinline__ void mm(Acc<M> &acc, const float *A, int lda, const float *B, int ldb, int K) {
    constexpr int RM = Acc<M>::RM;
    const int tid = threadIdx.x;
    const int m0 = RM * (tid >> 4), n0 = 4 * (tid & 15);
    if constexpr (!A_COL) {
#pragma unroll 2
        for (int k4 = 0; k4 < K; k4 += 4) {
            float4 a4[RM], b4[4];
#pragma unroll
            for (int i = 0; i < RM; ++i) a4[i] = *reinterpret_cast<const float4 *>(A + (size_t)(m0 + i) * lda + k4);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) b4[kk] = *reinterpret_cast<const float4 *>(B + (size_t)(k4 + kk) * ldb + n0);
#pragma unroll
            for (int i = 0; i < RM; ++i) {
                const float av[4] = {a4[i].x, a4[i].y, a4[i].z, a4[i].w};
#pragma unroll
                for (int kk = 0; kk < 4; ++kk) {
                    acc.c[i][0] = fmaf(av[kk], b4[kk].x, acc.c[i][0]);
                    acc.c[i][1] = fmaf(av[kk], b4[kk].y, acc.c[i][1]);
                    acc.c[i][2] = fmaf(av[kk], b4[kk].z, acc.c[i][2]);
                    acc.c[i][3] = fmaf(av[kk], b4[kk].w, acc.c[i][3]);
                }
            }
        }
        return;
    }
    float4 bn = *reinterpret_cast<const float4 *>(B + n0);
    float an[RM];
    load_a<M, A_COL>(an, A, lda, 0, m0);
#pragma unroll 4
    for (int k = 0; k < K; ++k) {
        const float4 b4 = bn;
        float av[RM];
#pragma unroll
        for (int i = 0; i < RM; ++i) av[i] = an[i];
        if (k + 1 < K) {
            bn = *reinterpret_cast<const float4 *>(B + (size_t)(k + 1) * ldb + n0);
            load_a<M, A_COL>(an, A, lda, k + 1, m0);
        }
#pragma unroll
        for (int i = 0; i < RM; ++i) {
            acc.c[i][0] = fmaf(av[i], b4.x, acc.c[i][0]);
            acc.c[i][1] = fmaf(av[i], b4.y, acc.c[i][1]);
            acc.c[i][2] = fmaf(av[i], b4.z, acc.c[i][2]);
            acc.c[i][3] = fmaf(av[i], b4.w, acc.c[i][3]);
        }
    }
}

// store the accumulator row-major (C[m * ldc + n]) or transposed (C[n * ldc + m])
template <int M>
__device__ __forceinline__ void put(const Acc<M> &acc, float *C, int ldc, bool transposed) {
    constexpr int RM = Acc<M>::RM;
    const int tid = threadIdx.x;
    const int m0 = RM * (tid >> 4), n0 = 4 * (tid & 15);
#pragma unroll
    for (int i = 0; i < RM; ++i) {
        if (!transposed) {
            *reinterpret_cast<float4 *>(C + (size_t)(m0 + i) * ldc + n0) =
                make_float4(acc.c[i][0], acc.c[i][1], acc.c[i][2], acc.c[i][3]);
        } else {
#pragma unroll
            for (int j = 0; j < 4; ++j) C[(size_t)(n0 + j) * ldc + m0 + i] = acc.c[i][j];
        }
    }
}

// shared-memory map of the gradient kernel (floats)
constexpr int SZ64 = 64 * LD, SZ32 = 32 * LD;
constexpr int O_AR = 0;                 // [64][LD] a' rows 0-31, r' rows 32-63 (token-major)
constexpr int O_BKT = O_AR + SZ64;      // [64 j][LD] b- (cols 0-31), k- (cols 32-63) (channel-major)
constexpr int O_X1 = O_BKT + SZ64;      // SG^T [j][i], then dS^T, then [b-; k-] token-major
constexpr int O_DZY = O_X1 + SZ64;      // [64][LD] dZ rows 0-31, dY rows 32-63
constexpr int O_UVT = O_DZY + SZ64;     // [64 i][LD] U (cols 0-31), V (cols 32-63) (channel-major)
constexpr int O_LB = O_UVT + SZ64;      // [L_ab L_ak; L_rb L_rk], then the dL block
constexpr int O_X2 = O_LB + SZ64;       // SG [i][j], then dS [i][j]
constexpr int O_V = O_X2 + SZ64;        // V [s][i], then dU
constexpr int O_Z = O_V + SZ32;         // Z, then da_{t} a_t for q
constexpr int O_T = O_Z + SZ32;         // T [32][LDS]
constexpr int O_ZS = O_T + 32 * LDS;    // [16][16] scratch of the inverse
constexpr int O_P = O_ZS + 256;         // p [33][64]
constexpr int O_RAW = O_P + 33 * kN;    // r w k a b, [5][32][64]
constexpr int O_Q = O_RAW + 5 * L * kN; // q [32][64]
constexpr int SMEM_FLOATS = O_Q + L * kN;
constexpr size_t SMEM_BYTES = (size_t)SMEM_FLOATS * sizeof(float);

}  // namespace bwdc

// ---------------------------------------------------------------------------
// Gradients of one chunk (one CTA per chunk, 256 threads), from S_in(c),
// S_out(c) (the next checkpoint, or the final state) and dS_out(c).
// ---------------------------------------------------------------------------
template <typename InT, typename GradT>
__global__ void __launch_bounds__(bwdc::NT, 1)
bwd_chunk_kernel(int T, int H, const InT *__restrict__ r, const InT *__restrict__ w, const InT *__restrict__ k,
                 const InT *__restrict__ v, const InT *__restrict__ a, const InT *__restrict__ b,
                 const InT *__restrict__ dy, const float *__restrict__ ckpt, const float *__restrict__ sfin,
                 const float *__restrict__ dS_out, GradT *__restrict__ dr, GradT *__restrict__ dw,
                 GradT *__restrict__ dk, GradT *__restrict__ dv, GradT *__restrict__ da,
                 GradT *__restrict__ db) {
    using namespace bwdc;
    extern __shared__ __align__(16) unsigned char dsmem[];
    float *sm = reinterpret_cast<float *>(dsmem);
    const int tid = threadIdx.x;
    const int nck = (T + L - 1) / L;
    const int head = blockIdx.x / nck, c = blockIdx.x % nck;     // chunk-major within a head
    const int bb = head / H, h = head % H;
    const int t0 = c * L, Lc = min(L, T - t0);
    const size_t tok_stride = (size_t)H * kN;
    const size_t base = (((size_t)bb * T + t0) * H + h) * kN;       // token t0 of this head
    const float *S_in = ckpt + ((size_t)head * nck + c) * kN * kN;
    const float *S_out = c + 1 < nck ? ckpt + ((size_t)head * nck + c + 1) * kN * kN : sfin + (size_t)head * kN * kN;
    const float *dSo = dS_out + ((size_t)head * nck + c) * kN * kN;
    float *AR = sm + O_AR, *BKT = sm + O_BKT, *X1 = sm + O_X1, *DZY = sm + O_DZY, *UVT = sm + O_UVT;
    float *LB = sm + O_LB, *X2 = sm + O_X2, *VB = sm + O_V, *ZB = sm + O_Z, *TB = sm + O_T, *ZS = sm + O_ZS;
    float *P = sm + O_P, *RAW = sm + O_RAW, *Q = sm + O_Q;
    auto raw = [&](int ten, int t, int j) -> float & { return RAW[(ten * L + t) * kN + j]; };   // r w k a b
    const int m0_64 = 4 * (tid >> 4), m0_32 = 2 * (tid >> 4), n0 = 4 * (tid & 15);

    // 1. every global read of the chunk is issued here: the states (thread ->
    //    float4 u of element 4 (tid + 256 u)) stay in registers until used
    float4 s_in[4], ds_o[4], s_ou[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int x = 4 * (tid + NT * u);
        s_in[u] = __ldcg(reinterpret_cast<const float4 *>(S_in + x));
        ds_o[u] = __ldcg(reinterpret_cast<const float4 *>(dSo + x));
        s_ou[u] = __ldcg(reinterpret_cast<const float4 *>(S_out + x));
    }
    //    inputs of the chunk (rows past the end: no-op tokens, w = 1), four
    //    consecutive channels per thread and pass
    for (int x = 4 * tid; x < L * kN; x += 4 * NT) {
        const int t = x >> 6, j = x & 63;
        const bool ok = t < Lc;
        const size_t g = base + (size_t)t * tok_stride + j;
        const float4 z4 = make_float4(0.f, 0.f, 0.f, 0.f);
        const float4 r4 = ok ? load4(r + g) : z4, w4 = ok ? load4(w + g) : make_float4(1.f, 1.f, 1.f, 1.f);
        const float4 k4 = ok ? load4(k + g) : z4, a4 = ok ? load4(a + g) : z4, b4 = ok ? load4(b + g) : z4;
        const float4 v4 = ok ? load4(v + g) : z4, y4 = ok ? load4(dy + g) : z4;
        *reinterpret_cast<float4 *>(&raw(0, t, j)) = r4;
        *reinterpret_cast<float4 *>(&raw(1, t, j)) = w4;
        *reinterpret_cast<float4 *>(&raw(2, t, j)) = k4;
        *reinterpret_cast<float4 *>(&raw(3, t, j)) = a4;
        *reinterpret_cast<float4 *>(&raw(4, t, j)) = b4;
        *reinterpret_cast<float4 *>(VB + t * LD + j) = v4;
        const float vv[4] = {v4.x, v4.y, v4.z, v4.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) UVT[(j + e) * LD + 32 + t] = vv[e];
        *reinterpret_cast<float4 *>(DZY + (32 + t) * LD + j) = y4;
    }
    __syncthreads();
    // 2. suffix decay products, one thread per channel
    if (tid < kN) {
        float pp = 1.f;
        P[L * kN + tid] = 1.f;
        for (int t = L - 1; t >= 0; --t) {
            pp *= raw(1, t, tid);
            P[t * kN + tid] = pp;
        }
        if (pp < kMinDecay) raise_status(WKV7_ERR_RANGE);
    }
    __syncthreads();
    // 3. scaled operands, and SG^T = (S_in diag(G))^T
    for (int x = tid; x < L * kN; x += NT) {
        const int t = x >> 6, j = x & 63;
        const float pt = P[t * kN + j], pn = P[(t + 1) * kN + j];
        AR[t * LD + j] = raw(3, t, j) / pt;
        AR[(32 + t) * LD + j] = raw(0, t, j) / pn;
        BKT[j * LD + t] = raw(4, t, j) * pn;
        BKT[j * LD + 32 + t] = raw(2, t, j) * pn;
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int x = 4 * (tid + NT * u), i = x >> 6, j = x & 63;
        const float sv[4] = {s_in[u].x * P[j], s_in[u].y * P[j + 1], s_in[u].z * P[j + 2], s_in[u].w * P[j + 3]};
#pragma unroll
        for (int e = 0; e < 4; ++e) X1[(j + e) * LD + i] = sv[e];
        *reinterpret_cast<float4 *>(X2 + i * LD + j) = make_float4(sv[0], sv[1], sv[2], sv[3]);
    }
    __syncthreads();
    // 4. [L_ab L_ak; L_rb L_rk] = [a'; r'] [b-; k-]^T, masked
    {
        Acc<64> acc;
        acc.zero();
        mm<64, false>(acc, AR, LD, BKT, LD, kN);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int m = m0_64 + i, n = n0 + jj, t = m & 31, s = n & 31;
                if (m < 32 ? s >= t : s > t) acc.c[i][jj] = 0.f;
            }
        put(acc, LB, LD, false);
    }
    __syncthreads();
    // 5. T = (I - L_ab)^{-1}: two 16x16 diagonal blocks by forward substitution
    //    (one column per lane of warp 0), then T21 = T22 L21 T11
    if (tid < 32) {
        const int blk = tid >> 4, s = tid & 15, o = 16 * blk;
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = e == s ? 1.f : 0.f;
#pragma unroll
        for (int m = 0; m < 15; ++m) {
            const float x = acc[m];
#pragma unroll
            for (int e = m + 1; e < 16; ++e) acc[e] = fmaf(LB[(o + e) * LD + o + m], x, acc[e]);
        }
#pragma unroll
        for (int e = 0; e < 16; ++e) TB[(o + e) * LDS + o + s] = acc[e];
    } else if (tid < 64) {
        const int s = tid & 31;
        if (s < 16)
#pragma unroll
            for (int e = 0; e < 16; ++e) TB[e * LDS + 16 + s] = 0.f;
    }
    __syncthreads();
    {
        const int t = tid >> 4, s = tid & 15;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) acc = fmaf(LB[(16 + t) * LD + m], TB[m * LDS + s], acc);
        ZS[t * 16 + s] = acc;
    }
    __syncthreads();
    {
        const int t = tid >> 4, s = tid & 15;
        float acc = 0.f;
#pragma unroll
        for (int m = 0; m < 16; ++m) acc = fmaf(TB[(16 + t) * LDS + 16 + m], ZS[m * 16 + s], acc);
        TB[(16 + t) * LDS + s] = acc;
    }
    __syncthreads();
    // 6. Z = a' SG^T + L_ak V
    {
        Acc<32> acc;
        acc.zero();
        mm<32, false>(acc, AR, LD, X1, LD, kN);
        mm<32, false>(acc, LB + 32, LD, VB, LD, L);
        put(acc, ZB, LD, false);
    }
    __syncthreads();
    // 7. U = T Z, stored channel-major next to V;  dS^T replaces SG^T
    {
        Acc<32> acc;
        acc.zero();
        mm<32, false>(acc, TB, LDS, ZB, LD, L);
        put(acc, UVT, LD, true);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int x = 4 * (tid + NT * u), i = x >> 6, j = x & 63;
        X1[j * LD + i] = ds_o[u].x;
        X1[(j + 1) * LD + i] = ds_o[u].y;
        X1[(j + 2) * LD + i] = ds_o[u].z;
        X1[(j + 3) * LD + i] = ds_o[u].w;
    }
    __syncthreads();
    // 8. dU = b- dS^T + L_rb^T dY  (into VB)
    {
        Acc<32> acc;
        acc.zero();
        mm<32, true>(acc, BKT, LD, X1, LD, kN);
        mm<32, true>(acc, LB + 32 * LD, LD, DZY + 32 * LD, LD, L);
        put(acc, VB, LD, false);
    }
    __syncthreads();
    // 9. dZ = T^T dU  (into DZY rows 0-31)
    {
        Acc<32> acc;
        acc.zero();
        mm<32, true>(acc, TB, LDS, VB, LD, L);
        put(acc, DZY, LD, false);
    }
    __syncthreads();
    // 10. dV = k- dS^T + L_rk^T dY + L_ak^T dZ  -> dv
    {
        Acc<32> acc;
        acc.zero();
        mm<32, true>(acc, BKT + 32, LD, X1, LD, kN);
        mm<32, true>(acc, LB + 32 * LD + 32, LD, DZY + 32 * LD, LD, L);
        mm<32, true>(acc, LB + 32, LD, DZY, LD, L);
#pragma unroll
        for (int i = 0; i < 2; ++i) {
            const int s = m0_32 + i;
            if (s < Lc)
                store4(dv + base + (size_t)s * tok_stride + n0,
                       make_float4(acc.c[i][0], acc.c[i][1], acc.c[i][2], acc.c[i][3]));
        }
    }
    __syncthreads();
    // 11. [dL_ab dL_ak; dL_rb dL_rk] = [dZ; dY] [U; V]^T, masked (into LB)
    {
        Acc<64> acc;
        acc.zero();
        mm<64, false>(acc, DZY, LD, UVT, LD, kN);
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                const int m = m0_64 + i, n = n0 + jj, t = m & 31, s = n & 31;
                if (m < 32 ? s >= t : s > t) acc.c[i][jj] = 0.f;
            }
        put(acc, LB, LD, false);   // the L block was last read in step 10
    }
    // 12. [b-; k-] token-major (X1); SG is already in X2
    for (int x = tid; x < kN * kN; x += NT) {
        const int i = x >> 6, j = x & 63;
        X1[i * LD + j] = BKT[j * LD + i];
    }
    __syncthreads();
    // 13. da, dr: [dZ; dY] SG + dL [b-; k-], then the decay factors; q terms
    {
        Acc<64> acc;
        acc.zero();
        mm<64, false>(acc, DZY, LD, X2, LD, kN);
        mm<64, false>(acc, LB, LD, X1, LD, kN);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = m0_64 + i, t = m & 31;
            float o[4];
            if (m < 32) {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    o[jj] = acc.c[i][jj] / P[t * kN + n0 + jj];
                    ZB[t * LD + n0 + jj] = o[jj] * raw(3, t, n0 + jj);
                }
                if (t < Lc) store4(da + base + (size_t)t * tok_stride + n0, make_float4(o[0], o[1], o[2], o[3]));
            } else {
#pragma unroll
                for (int jj = 0; jj < 4; ++jj) {
                    o[jj] = acc.c[i][jj] / P[(t + 1) * kN + n0 + jj];
                    Q[t * kN + n0 + jj] = o[jj] * raw(0, t, n0 + jj);
                }
                if (t < Lc) store4(dr + base + (size_t)t * tok_stride + n0, make_float4(o[0], o[1], o[2], o[3]));
            }
        }
    }
    __syncthreads();
    // 14. dS row-major (X2)
#pragma unroll
    for (int u = 0; u < 4; ++u) {
        const int x = 4 * (tid + NT * u), i = x >> 6, j = x & 63;
        *reinterpret_cast<float4 *>(X2 + i * LD + j) = ds_o[u];
    }
    __syncthreads();
    // 15. db, dk: [U; V] dS + dL^T [a'; r'], times p_{s+1}; q terms
    {
        Acc<64> acc;
        acc.zero();
        mm<64, true>(acc, UVT, LD, X2, LD, kN);
        mm<64, true>(acc, LB, LD, AR, LD, kN);
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int m = m0_64 + i, s = m & 31;
            const int ten = m < 32 ? 4 : 2;   // b or k
            float o[4];
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) {
                o[jj] = acc.c[i][jj] * P[(s + 1) * kN + n0 + jj];
                atomicAdd(&Q[s * kN + n0 + jj], -o[jj] * raw(ten, s, n0 + jj));
            }
            if (s < Lc) store4((m < 32 ? db : dk) + base + (size_t)s * tok_stride + n0, make_float4(o[0], o[1], o[2], o[3]));
        }
    }
    // 16. the last token's decay also scales S_out: q_{Lc-1} += sum_i S_out dS.
    //     A thread's four float4 share columns 4 (tid & 15) .. +3; lanes l and
    //     l + 16 too: sum those first, then one atomic per column and warp.
    {
        float cs[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            cs[0] = fmaf(s_ou[u].x, ds_o[u].x, cs[0]);
            cs[1] = fmaf(s_ou[u].y, ds_o[u].y, cs[1]);
            cs[2] = fmaf(s_ou[u].z, ds_o[u].z, cs[2]);
            cs[3] = fmaf(s_ou[u].w, ds_o[u].w, cs[3]);
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 16);
        if ((tid & 31) < 16) {
            float *qr = Q + (Lc - 1) * kN + 4 * (tid & 15);
#pragma unroll
            for (int e = 0; e < 4; ++e) atomicAdd(qr + e, cs[e]);
        }
    }
    __syncthreads();
    // 17. dw_m = sum_{t >= m} q_t / w_m,  q_t = Q_t + da_{t+1} a_{t+1}
    if (tid < kN) {
        const int j = tid;
        float run = 0.f;
        for (int t = Lc - 1; t >= 0; --t) {
            run += Q[t * kN + j] + (t + 1 < Lc ? ZB[(t + 1) * LD + j] : 0.f);
            dw[base + (size_t)t * tok_stride + j] = from_f32<GradT>(run / raw(1, t, j));
        }
    }
}

size_t bwd_chunk_ckpt_bytes(int B, int T, int H) {
    const size_t nck = ((size_t)T + bwdc::L - 1) / bwdc::L;
    return (size_t)B * H * nck * kN * kN * sizeof(float);
}

cudaError_t bwd_chunk_tc(int B, int T, int H, wkv7_dtype g_dt, const void *r, const void *w, const void *k,
                         const void *v, const void *a, const void *b, const void *dy, const float *ckpt,
                         const float *sfin, const float *dS_out, void *dr, void *dw, void *dk, void *dv, void *da,
                         void *db, long long wait_limit, cudaStream_t st);

static cudaError_t launch_combine(int B, int H, int nsteps, const float *s0, bool s0_eye, const float *e_base,
                                  long long e_stride, const float *m_base, long long m_stride, float *out,
                                  long long out_stride, cudaStream_t st, bool transpose_m);   // fwd_chunk.cu

size_t dstate_scratch_bytes(int B, int H, int nseg) {
    return nseg > 1 ? 3ULL * nseg * B * H * kN * kN * sizeof(float) : 0;
}

namespace {

// One launch of the sweep kernel: nz segments from seg0, all heads; rpt rows
// per thread and lpr lanes per row (rpt 1 splits a head over two CTAs).
template <typename I>
cudaError_t launch_dstate(int rpt, int lpr, bool dual, int heads, int T, int H, int t_seg, int seg0, int nz,
                          const void *r, const void *w, const void *a, const void *b, const void *dy,
                          const float *g_in, long long g_in_zs, float *dS_out, float *g_out, long long g_out_zs,
                          int g_out_nz, float *m_out, long long m_zs, cudaStream_t st) {
    const size_t smem = 2 * 5 * bwdc::L * kN * sizeof(I);
    if (lpr != 8) lpr = 4;
    if (lpr == 8) rpt = 4;
    if (rpt == 4 && lpr == 4 && dual) rpt = 2;     // eight rows of two states in 16 columns would spill
    const int split = rpt == 1 ? 2 : 1;
    const unsigned grid = (unsigned)((size_t)nz * heads * split);
    const int threads = lpr * kN / (split * rpt);
#define WKV7_DSTATE(R, P, D)                                                                                 \
    do {                                                                                                     \
        auto kern = bwd_dstate_kernel<I, R, P, D>;                                                           \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);    \
        if (e != cudaSuccess) return e;                                                                      \
        kern<<<grid, threads, smem, st>>>(T, t_seg, seg0, nz, (const I *)r, (const I *)w, (const I *)a,     \
                                          (const I *)b, (const I *)dy, H, g_in, g_in_zs, dS_out, g_out,     \
                                          g_out_zs, g_out_nz, m_out, m_zs);                                  \
    } while (0)
    if (lpr == 8) {
        if (dual) WKV7_DSTATE(4, 8, true);
        else WKV7_DSTATE(4, 8, false);
    } else if (rpt == 1) {
        if (dual) WKV7_DSTATE(1, 4, true);
        else WKV7_DSTATE(1, 4, false);
    } else if (rpt == 4) {
        WKV7_DSTATE(4, 4, false);
    } else {
        if (dual) WKV7_DSTATE(2, 4, true);
        else WKV7_DSTATE(2, 4, false);
    }
#undef WKV7_DSTATE
    return cudaGetLastError();
}

}  // namespace

// The sweep's plan: segments (whole chunks, all non-empty) and rows per
// thread, for B*H heads of T tokens.
struct DstatePlan {
    int nseg = 1, t_seg = 0, rpt = 2, lpr = 4;
};

DstatePlan dstate_split(int T, int nseg_want, int rpt, int lpr = 4) {
    DstatePlan p;
    const int chunks = (T + bwdc::L - 1) / bwdc::L;
    const int want = std::max(1, std::min(nseg_want, chunks));
    const int per = (chunks + want - 1) / want;
    p.t_seg = per * bwdc::L;
    p.nseg = (chunks + per - 1) / per;
    p.rpt = rpt;
    p.lpr = lpr;
    return p;
}

// Estimated time (ns) of one sweep launch of n CTAs over `steps` tokens.  A
// step of a CTA alone on its SM is latency-bound; each further co-resident
// CTA adds its issue time (for the two-warp CTAs of rpt 4, from the third on);
// CTAs beyond the resident ones run in later waves.  Fitted on B200 (bf16
// inputs; B = 1 .. 16, H = 32, T = 4096 .. 65536).
static double dstate_launch_ns(long long n, long long steps, int rpt, int lpr, bool dual, bool f32, int sms) {
    double lat, add;
    long long free_k = 1;
    if (lpr == 8) {
        lat = 197.0;
        add = 120.0;
    } else if (rpt == 1) {
        lat = dual ? 198.0 : 156.0;
        add = dual ? 115.0 : 156.0;
    } else if (rpt == 2) {
        lat = dual ? 252.0 : 221.0;
        add = dual ? 191.0 : 109.0;
    } else {
        lat = 306.0;
        add = 110.0;
        free_k = 2;
    }
    const int res = f32 ? 2 : (rpt == 2 && dual ? 4 : 5);    // shared memory, registers
    const long long per_sm = (n + sms - 1) / sms;
    const long long waves = (per_sm + res - 1) / res;
    const long long k = std::min<long long>(per_sm, res);
    return (double)waves * (double)steps * (lat + add * (double)std::max<long long>(0, k - free_k));
}

// The plan with the lowest estimated time whose scratch fits scratch_cap
// bytes: rpt 1, 2 or 4 rows per thread with four lanes per row, or 4 rows
// with eight lanes (those two one-pass only), nseg = 1 or a split into
// segments of at least two chunks.
// need_dS: dS at every chunk end is wanted (the backward), else ds0 alone.
DstatePlan dstate_plan(int B, int T, int H, int sms, bool f32, bool need_dS, size_t scratch_cap,
                       double *est_ns = nullptr) {
    const long long heads = (long long)B * H;
    const int chunks = (T + bwdc::L - 1) / bwdc::L;
    if (sms <= 0) sms = 148;
    constexpr double kCombineStepNs = 3000.0, kLaunchNs = 4000.0;
    DstatePlan best;
    double best_ns = 0.0;
    for (int variant = 0; variant < 4; ++variant) {
        const int rpt = variant == 0 ? 1 : variant == 1 ? 2 : 4, lpr = variant == 3 ? 8 : 4;
        const long long per_head = rpt == 1 ? 2 : 1;
        for (int want = 1; want <= (rpt == 4 ? 1 : std::min(64, std::max(1, chunks / 2))); ++want) {
            const DstatePlan p = dstate_split(T, want, rpt, lpr);
            if (p.nseg != want) continue;
            if (p.nseg > 1 && dstate_scratch_bytes(B, H, p.nseg) > scratch_cap) break;
            const int n = p.nseg;
            double ns;
            if (n == 1) {
                ns = dstate_launch_ns(heads * per_head, T, rpt, lpr, false, f32, sms);
            } else if (need_dS) {
                const long long ctas = (n - 1) * heads * per_head;
                ns = dstate_launch_ns(ctas, p.t_seg, rpt, lpr, n > 2, f32, sms) +
                     dstate_launch_ns(ctas, p.t_seg, rpt, lpr, false, f32, sms) + kCombineStepNs * (n - 2) +
                     kLaunchNs * (n > 2 ? 2 : 1);
            } else {
                ns = dstate_launch_ns(n * heads * per_head, p.t_seg, rpt, lpr, true, f32, sms) +
                     kCombineStepNs * (n - 1) + kLaunchNs;
            }
            if (best_ns == 0.0 || ns < 0.97 * best_ns) {
                best = p;
                best_ns = ns;
            }
        }
    }
    if (est_ns) *est_ns = best_ns;
    return best;
}

double bwd_dchain_ns(int B, int T, int H, int sms);   // bwd_dchain.cu

// Whether the transition chain (bwd_dchain.cu) beats the per-token sweep for
// dS at every chunk end, bf16 inputs, the sweep given scratch_cap bytes of
// scratch.
bool bwd_use_dchain(int B, int T, int H, int sms, size_t scratch_cap) {
    double sweep_ns = 0.0;
    dstate_plan(B, T, H, sms, false, true, scratch_cap, &sweep_ns);
    return bwd_dchain_ns(B, T, H, sms) < 0.9 * sweep_ns;
}

// Scratch of the plan dstate_plan picks with room to spare, for either input
// dtype (workspace sizes do not depend on it).
size_t dstate_scratch_for(int B, int T, int H, int sms, bool need_dS) {
    size_t need = 0;
    for (bool f32 : {false, true}) {
        const DstatePlan p = dstate_plan(B, T, H, sms, f32, need_dS, (size_t)-1);
        need = std::max(need, dstate_scratch_bytes(B, H, p.nseg));
    }
    return need;
}

// dL/dS at every chunk end (into dS_out, skipped when it is null) and ds0, by
// the reverse sweep of the state gradient; reads r, w, a, b, dy only.  With
// nseg > 1 segments (scratch: dstate_scratch_bytes), the segments' dual runs,
// a chain of their summaries for the entry adjoints, and (for dS_out) output
// runs of all segments but the last.
template <typename I>
cudaError_t bwd_dstate_run(int B, int T, int H, const DstatePlan &p, const void *r, const void *w, const void *a,
                           const void *b, const void *dy, const float *dsT, float *dS_out, float *ds0,
                           float *scratch, cudaStream_t st) {
    const int heads = B * H, n = p.nseg;
    if (n <= 1)
        return launch_dstate<I>(p.rpt, p.lpr, false, heads, T, H, std::max(p.t_seg, T), 0, 1, r, w, a, b, dy, dsT, 0,
                                dS_out, ds0, 0, 1, nullptr, 0, st);
    const long long zs = (long long)heads * kN * kN;
    float *FA = scratch, *MT = scratch + n * zs, *ADJ = scratch + 2 * n * zs;
    cudaError_t e;
    if (!dS_out) {
        // every segment summarised (the last one from dsT), then one chain to ds0
        e = launch_dstate<I>(p.rpt, p.lpr, true, heads, T, H, p.t_seg, 0, n, r, w, a, b, dy, dsT, 0, nullptr, FA, zs, n,
                             MT, zs, st);
        if (e != cudaSuccess) return e;
        return launch_combine(B, H, n - 1, FA + (n - 1) * zs, false, FA + (n - 2) * zs, -zs, MT + (n - 2) * zs, -zs,
                              ds0, 0, st, false);
    }
    // pass 1: segments 1..n-1, the last as an output run from dsT
    e = launch_dstate<I>(p.rpt, p.lpr, n > 2, heads, T, H, p.t_seg, 1, n - 1, r, w, a, b, dy, dsT, 0, dS_out, FA + zs, zs,
                         n - 1, MT + zs, zs, st);
    if (e != cudaSuccess) return e;
    // pass 2: dL/dS at the end of segments 0..n-2: adj[k] = adj[k+1] M_k^T + F_k
    const float *entry = FA + zs;
    if (n > 2) {
        e = launch_combine(B, H, n - 2, FA + (n - 1) * zs, false, FA + (n - 2) * zs, -zs, MT + (n - 2) * zs, -zs,
                           ADJ + (n - 1) * zs, -zs, st, false);
        if (e != cudaSuccess) return e;
        entry = ADJ + zs;
    }
    // pass 3: output runs of segments 0..n-2; segment 0 ends with ds0
    return launch_dstate<I>(p.rpt, p.lpr, false, heads, T, H, p.t_seg, 0, n - 1, r, w, a, b, dy, entry, zs, dS_out, ds0, 0,
                            1, nullptr, 0, st);
}

cudaError_t bwd_dstate_plan(int B, int T, int H, wkv7_dtype in_dt, const DstatePlan &p, const void *r,
                            const void *w, const void *a, const void *b, const void *dy, const float *dsT,
                            float *dS_out, float *ds0, float *scratch, cudaStream_t st) {
    return in_dt == WKV7_F32
               ? bwd_dstate_run<float>(B, T, H, p, r, w, a, b, dy, dsT, dS_out, ds0, scratch, st)
               : bwd_dstate_run<__nv_bfloat16>(B, T, H, p, r, w, a, b, dy, dsT, dS_out, ds0, scratch, st);
}

// The sweep under the cost model's plan, within scratch_bytes of scratch.
cudaError_t bwd_dstate(int B, int T, int H, wkv7_dtype in_dt, const void *r, const void *w, const void *a,
                       const void *b, const void *dy, const float *dsT, float *dS_out, float *ds0, float *scratch,
                       size_t scratch_bytes, int sms, cudaStream_t st) {
    const DstatePlan p =
        dstate_plan(B, T, H, sms, in_dt == WKV7_F32, dS_out != nullptr, scratch ? scratch_bytes : 0);
    return bwd_dstate_plan(B, T, H, in_dt, p, r, w, a, b, dy, dsT, dS_out, ds0, scratch, st);
}

// The input gradients of every chunk from its checkpoint, the next one (or
// the final state) and dS at its end: tensor cores for bf16 inputs, fp32
// CUDA-core products for fp32 inputs.
cudaError_t bwd_chunk_grads(int B, int T, int H, wkv7_dtype in_dt, wkv7_dtype g_dt, const void *r, const void *w,
                            const void *k, const void *v, const void *a, const void *b, const void *dy,
                            const float *ckpt, const float *sfin, const float *dS_out, void *dr, void *dw, void *dk,
                            void *dv, void *da, void *db, long long wait_limit, cudaStream_t st) {
    using namespace bwdc;
    const int heads = B * H, nck = (T + L - 1) / L;
    if (in_dt == WKV7_BF16)
        return bwd_chunk_tc(B, T, H, g_dt, r, w, k, v, a, b, dy, ckpt, sfin, dS_out, dr, dw, dk, dv, da, db,
                            wait_limit, st);
    const dim3 grid((unsigned)((size_t)heads * nck));
#define WKV7_CHUNK_BWD(I, G)                                                                                 \
    do {                                                                                                     \
        auto kern = bwd_chunk_kernel<I, G>;                                                                  \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)SMEM_BYTES); \
        if (e != cudaSuccess) return e;                                                                      \
        kern<<<grid, NT, SMEM_BYTES, st>>>(T, H, (const I *)r, (const I *)w, (const I *)k, (const I *)v,    \
                                           (const I *)a, (const I *)b, (const I *)dy, ckpt, sfin, dS_out,  \
                                           (G *)dr, (G *)dw, (G *)dk, (G *)dv, (G *)da, (G *)db);           \
    } while (0)
    if (in_dt == WKV7_F32 && g_dt == WKV7_F32) WKV7_CHUNK_BWD(float, float);
    else if (in_dt == WKV7_F32) WKV7_CHUNK_BWD(float, __nv_bfloat16);
    else if (g_dt == WKV7_F32) WKV7_CHUNK_BWD(__nv_bfloat16, float);
    else WKV7_CHUNK_BWD(__nv_bfloat16, __nv_bfloat16);
#undef WKV7_CHUNK_BWD
    return cudaGetLastError();
}

cudaError_t bwd_dchain(int B, int T, int H, const void *dy, const uint4 *mq, const float *dsT, float *dS_out,
                       float *ds0, long long wait_limit, cudaStream_t st);   // bwd_dchain.cu

// dS at every chunk end (the transition chain when the checkpoint pass
// exported the chunks' transitions mq, bf16 inputs; else the sweep), then the
// chunk gradients.
cudaError_t bwd_chunked(int B, int T, int H, wkv7_dtype in_dt, wkv7_dtype g_dt, const void *r, const void *w,
                        const void *k, const void *v, const void *a, const void *b, const void *dy,
                        const float *dsT, const float *ckpt, const float *sfin, float *dS_out, void *dr,
                        void *dw, void *dk, void *dv, void *da, void *db, float *ds0, float *scratch,
                        size_t scratch_bytes, int sms, long long wait_limit, cudaStream_t st,
                        const uint4 *mq) {
    cudaError_t e = (mq != nullptr && in_dt == WKV7_BF16)
                        ? bwd_dchain(B, T, H, dy, mq, dsT, dS_out, ds0, wait_limit, st)
                        : bwd_dstate(B, T, H, in_dt, r, w, a, b, dy, dsT, dS_out, ds0, scratch, scratch_bytes, sms, st);
    if (e != cudaSuccess) return e;
    return bwd_chunk_grads(B, T, H, in_dt, g_dt, r, w, k, v, a, b, dy, ckpt, sfin, dS_out, dr, dw, dk, dv, da, db,
                           wait_limit, st);
}

}  // namespace wkv7
