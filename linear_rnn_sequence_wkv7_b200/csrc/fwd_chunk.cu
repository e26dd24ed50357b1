// Chunked WKV7 forward on the sm_100a tensor cores (tcgen05, TMEM accumulators).
//
// The pages state that RWKV-7 keeps training parallelisable (RWKV-7 "Goose"
// with Expressive Dynamic State Evolution, abstract) and cite chunk-wise
// parallelisation of the delta rule only by title; the algebra below is our
// own derivation from the recurrence
//     S_t = S_{t-1} (diag(w_t) + a_t b_t^T) + v_t k_t^T,   y_t = S_t r_t.
//
// Chunk of L = 32 tokens (local t, s in [0, 32)), entry state S (64 x 64,
// row i = value, column j = key), c_t = sum_{m<=t} log w_m per channel:
//   a~_t = a_t e^{c_{t-1}},  r~_t = r_t e^{c_t},  b^_t = b_t e^{-c_t},
//   k^_t = k_t e^{-c_t},     b-_t = b_t e^{c_31 - c_t},  k-_t = k_t e^{c_31 - c_t}
//   G     = [a~; r~] [b^; k^]^T                      Gram (64 x 64)
//   L_ab, L_ak = strictly lower parts of the a~ rows; L_rb, L_rk = lower parts
//                of the r~ rows (diagonal included)
//   T = (I - L_ab)^{-1},  P = T L_ak                 (32 x 32, CUDA cores, fp32)
//   W^T = A~^T T^T,  U~^T = V^T P^T                  (u_t = S w_t + u~_t)
//   M = diag(e^{c_31}) + W^T B-,  Q^T = R~^T + W^T L_rb^T
//   E = U~^T B- + V^T K-,  Y_loc^T = U~^T L_rb^T + V^T L_rk^T
//   S_out = S M + E,  Y^T = S Q^T + Y_loc^T          (state-dependent part)
//
// Precision: every tensor-core product uses bf16 hi/lo splits (x = hi + lo to
// 16 bits; three passes hi*hi + hi*lo + lo*hi, two when one side is an exact
// bf16 input such as v) with fp32 accumulation in TMEM.  A single tf32 or bf16
// pass is not accurate enough for the 2e-3 rms bound on this workload.
//
// Mapping: one CTA (128 threads, 4 warps) per (b, h); chunks are processed in
// order.  Per chunk: P0 (CUDA cores) builds the decayed operands from the
// token tile; R1 Gram; P1 masks, solves T and P; R2 W^T, U~^T; P2 stages
// them; R3 M', Q'^T, E, Y_loc^T; P3 finishes M and Q; R4 the state product
// accumulates onto [E | Y_loc^T]; P4 writes y and stages S_out as the next
// chunk's operand.  One thread issues the MMAs; completion is tracked by an
// mbarrier with a bounded wait.  The next chunk's tokens are fetched with
// cp.async while the current chunk runs.
//
// TMEM (256 columns, M=64 accumulators occupy lanes 16w..16w+15 of each warp
// quadrant; a second M=64 tile can sit at lane offset 16):
//   X: cols [0, 96)    G (64) -> M' (64) | Q'^T (32)
//   Y: cols [96, 128)  W^T at lane offset 0, U~^T at lane offset 16
//   Z: cols [128, 224) [E | Y_loc^T], then += S [M | Q^T]
#include "umma.cuh"

namespace wkv7 {

namespace chunk {

constexpr int L = 32;          // tokens per chunk
constexpr int NT = 128;        // threads per CTA
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_X = 0, COL_Y = 96, COL_Z = 128;

// shared memory map (bytes)
constexpr uint32_t IN = 0;                      // [6][32][64] bf16 token tile (r w k v a b)
constexpr uint32_t GA_HI = 24576, GA_LO = 32768;   // [64][64]: a~ rows 0..31, r~ rows 32..63
constexpr uint32_t R1 = 40960;                  // 16 KB, reused: GB | L/T/P scratch | W^T,U~^T | M
constexpr uint32_t GB_HI = R1, GB_LO = R1 + 8192;
constexpr uint32_t LAB = R1, LAK = R1 + 4096, TSM = R1 + 8192, PSM = R1 + 12288;   // fp32 [32][32]
constexpr uint32_t WT_HI = R1, WT_LO = R1 + 4096, UT_HI = R1 + 8192, UT_LO = R1 + 12288;  // [64][32]
constexpr uint32_t M_HI = R1, M_LO = R1 + 8192;  // [64][64]
constexpr uint32_t VB = 57344;                  // [32][64] exact bf16 v
constexpr uint32_t BBAR_HI = 61440, BBAR_LO = 65536, KBAR_HI = 69632, KBAR_LO = 73728;  // [32][64]
constexpr uint32_t RQ = 77824;                  // 8 KB, reused: cumsum fp32 [32][64] | T,P | Q
constexpr uint32_t CSUM = RQ;
constexpr uint32_t T_HI = RQ, T_LO = RQ + 2048, P_HI = RQ + 4096, P_LO = RQ + 6144;   // [32][32]
constexpr uint32_t Q_HI = RQ, Q_LO = RQ + 4096;  // [64][32]
constexpr uint32_t LRB_HI = 86016, LRB_LO = 88064, LRK_HI = 90112, LRK_LO = 92160;   // [32][32]
constexpr uint32_t S_HI = 94208, S_LO = 102400;  // [64][64]
constexpr uint32_t GAML = 110592;               // fp32 [64] e^{c_31}
constexpr uint32_t HALF = 110848;               // fp32 [64] partial cumsum
constexpr uint32_t MBAR = 111104;               // u64
constexpr uint32_t TMEM_SLOT = 111112;          // u32
constexpr uint32_t FLAG = 111116;               // u32 abort flag
constexpr uint32_t SMEM_BYTES = 111120;

constexpr long long kWaitCycles = 2000000000LL;   // ~1 s: far above any legitimate MMA round
constexpr float kMinLogDecay = -69.0f;            // per-chunk log decay floor (prod w >= 1e-30)

}  // namespace chunk

template <typename OutT>
__global__ void __launch_bounds__(chunk::NT, 1)
fwd_chunk_kernel(int T, int H, const __nv_bfloat16 *__restrict__ r, const __nv_bfloat16 *__restrict__ w,
                 const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
                 const __nv_bfloat16 *__restrict__ a, const __nv_bfloat16 *__restrict__ b,
                 const float *s0, OutT *__restrict__ y, float *sT) {
    using namespace chunk;
    using namespace umma;
    extern __shared__ __align__(1024) unsigned char sm[];
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, bb = blockIdx.y;
    const size_t tok_stride = (size_t)H * kN;
    const size_t base = ((size_t)bb * T * H + h) * kN;
    const size_t st_base = ((size_t)bb * H + h) * kN * kN;
    const int nchunks = (T + L - 1) / L;
    const __nv_bfloat16 *src[6] = {r, w, k, v, a, b};
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(sm + FLAG);
    const uint32_t mbar = sbase + MBAR;

    auto issue_chunk = [&](int c) {
        const int t0 = c * L;
        for (int x = tid; x < 6 * L * 8; x += NT) {
            const int ten = x >> 8, rem = x & 255, t = rem >> 3, ch = rem & 7;
            if (t0 + t < T)
                cp_async16(sm + IN + ((ten * L + t) * kN + ch * 8) * 2,
                           src[ten] + base + (size_t)(t0 + t) * tok_stride + ch * 8);
        }
        cp_async_commit();
    };

    // ---- set-up: barrier, TMEM, first tile, initial state operand ---------------
    if (tid == 0) {
        mbar_init(mbar, 1);
        *abort_flag = 0;
    }
    if (warp == 0) tmem_alloc(sbase + TMEM_SLOT, TMEM_COLS);
    issue_chunk(0);
    {
        // S operand: row i = tid >> 1, columns 32*(tid&1) .. +32
        const int i = tid >> 1, c0 = (tid & 1) * 32;
        for (int g = 0; g < 4; ++g) {
            float x[8];
            for (int e = 0; e < 8; ++e) x[e] = s0 ? s0[st_base + (size_t)i * kN + c0 + 8 * g + e] : 0.f;
            store8_split(sm + S_HI, sm + S_LO, cm_off(i, c0 + 8 * g, 64), x);
        }
    }
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + TMEM_SLOT);
    const uint32_t quad = (uint32_t)(32 * warp) << 16;   // this warp's TMEM lane quadrant
    uint32_t phase = 0;

    auto round_wait = [&]() -> bool {
        const bool ok = mbar_wait(mbar, phase, kWaitCycles);
        phase ^= 1u;
        if (!ok) *abort_flag = 1;
        __syncthreads();
        fence_after_sync();
        return *abort_flag == 0;
    };
    auto issue_begin = [&]() {   // all threads: publish smem writes / TMEM reads, then sync
        fence_smem_to_async();
        fence_before_sync();
        __syncthreads();
    };

    for (int c = 0; c < nchunks; ++c) {
        const int t0 = c * L;
        const int Lv = min(L, T - t0);
        cp_async_wait<0>();
        __syncthreads();

        // ---- P0a: cumulative log decay per channel ----------------------------------
        {
            const int j = tid & 63, half = tid >> 6;
            const __nv_bfloat16 *wv = reinterpret_cast<const __nv_bfloat16 *>(sm + IN) + (1 * L) * kN;
            float cs[16];
            float acc = 0.f;
#pragma unroll
            for (int q = 0; q < 16; ++q) {
                const int t = 16 * half + q;
                const float lw = (t < Lv) ? logf(__bfloat162float(wv[t * kN + j])) : 0.f;
                acc += lw;
                cs[q] = acc;
            }
            float *half_sum = reinterpret_cast<float *>(sm + HALF);
            if (half == 0) half_sum[j] = acc;
            __syncthreads();
            const float off = half ? half_sum[j] : 0.f;
            float *csum = reinterpret_cast<float *>(sm + CSUM);
#pragma unroll
            for (int q = 0; q < 16; ++q) csum[(16 * half + q) * kN + j] = cs[q] + off;
            if (half == 1) {
                const float c31 = cs[15] + off;
                reinterpret_cast<float *>(sm + GAML)[j] = expf(c31);
                if (c31 < kMinLogDecay) raise_status(WKV7_ERR_RANGE);
            }
        }
        __syncthreads();

        // ---- P0b: decayed operands of this chunk ------------------------------------
        {
            const int t = tid >> 2, jq = tid & 3;
            const float *csum = reinterpret_cast<const float *>(sm + CSUM);
            const bool valid = t < Lv;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
                const int j0 = 16 * jq + 8 * g;
                float xa[8], xr[8], xb[8], xk[8], xbb[8], xkb[8];
                const uint4 *row = reinterpret_cast<const uint4 *>(sm + IN);
                auto ld8 = [&](int ten, float *o) {
                    const uint4 u = row[((ten * L + t) * kN + j0) >> 3];
                    const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        o[2 * q] = valid ? __uint_as_float(uu[q] << 16) : 0.f;
                        o[2 * q + 1] = valid ? __uint_as_float(uu[q] & 0xffff0000u) : 0.f;
                    }
                };
                float rr[8], kk[8], aa[8], bv[8];
                ld8(0, rr);
                ld8(2, kk);
                ld8(4, aa);
                ld8(5, bv);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float ct = csum[t * kN + j0 + e];
                    const float cp = t > 0 ? csum[(t - 1) * kN + j0 + e] : 0.f;
                    const float c31 = csum[(L - 1) * kN + j0 + e];
                    const float einv = expf(-ct), ebar = expf(c31 - ct);
                    xa[e] = aa[e] * expf(cp);
                    xr[e] = rr[e] * expf(ct);
                    xb[e] = bv[e] * einv;
                    xk[e] = kk[e] * einv;
                    xbb[e] = bv[e] * ebar;
                    xkb[e] = kk[e] * ebar;
                }
                store8_split(sm + GA_HI, sm + GA_LO, cm_off(t, j0, 64), xa);
                store8_split(sm + GA_HI, sm + GA_LO, cm_off(L + t, j0, 64), xr);
                store8_split(sm + GB_HI, sm + GB_LO, cm_off(t, j0, 64), xb);
                store8_split(sm + GB_HI, sm + GB_LO, cm_off(L + t, j0, 64), xk);
                store8_split(sm + BBAR_HI, sm + BBAR_LO, cm_off(t, j0, 64), xbb);
                store8_split(sm + KBAR_HI, sm + KBAR_LO, cm_off(t, j0, 64), xkb);
                const uint4 vv = valid ? row[((3 * L + t) * kN + j0) >> 3] : make_uint4(0, 0, 0, 0);
                *reinterpret_cast<uint4 *>(sm + VB + cm_off(t, j0, 64)) = vv;
            }
        }
        __syncthreads();                      // token tile consumed
        if (c + 1 < nchunks) issue_chunk(c + 1);

        // ---- R1: Gram -------------------------------------------------------------
        issue_begin();
        if (tid == 0) {
            fence_after_sync();
            gemm_split(tmem + COL_X, op_k(sbase + GA_HI, sbase + GA_LO, 64), op_k(sbase + GB_HI, sbase + GB_LO, 64),
                       idesc_bf16(64, 64, 0, 0), 4, false);
            commit(mbar);
        }
        if (!round_wait()) break;

        // ---- P1: masks, T = (I - L_ab)^{-1}, P = T L_ak -------------------------------
        {
            float g[64];
#pragma unroll
            for (int q = 0; q < 4; ++q) tmem_ld16(tmem + quad + COL_X + 16 * q, *reinterpret_cast<float(*)[16]>(g + 16 * q));
            if (lane < 16) {
                const int rho = 16 * warp + lane;
                if (rho < L) {            // a~ row t: strictly lower L_ab, L_ak (fp32 scratch)
                    const int t = rho;
                    float *lab = reinterpret_cast<float *>(sm + LAB) + t * L;
                    float *lak = reinterpret_cast<float *>(sm + LAK) + t * L;
#pragma unroll
                    for (int s = 0; s < L; ++s) {
                        lab[s] = s < t ? g[s] : 0.f;
                        lak[s] = s < t ? g[L + s] : 0.f;
                    }
                } else {                  // r~ row t: lower L_rb, L_rk (B operands)
                    const int t = rho - L;
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        float xb[8], xk[8];
#pragma unroll
                        for (int e = 0; e < 8; ++e) {
                            const int s = 8 * q + e;
                            xb[e] = s <= t ? g[s] : 0.f;
                            xk[e] = s <= t ? g[L + s] : 0.f;
                        }
                        store8_split(sm + LRB_HI, sm + LRB_LO, cm_off(t, 8 * q, L), xb);
                        store8_split(sm + LRK_HI, sm + LRK_LO, cm_off(t, 8 * q, L), xk);
                    }
                }
            }
        }
        __syncthreads();
        if (warp < 2) {
            // lane s owns column s; warp 0 solves T, warp 1 solves P
            const float *lab = reinterpret_cast<const float *>(sm + LAB);
            float *out = reinterpret_cast<float *>(sm + (warp == 0 ? TSM : PSM));
            const float *rhs = reinterpret_cast<const float *>(sm + LAK);
            const int s = lane;
            for (int t = 0; t < L; ++t) {
                float acc0 = warp == 0 ? (t == s ? 1.f : 0.f) : rhs[t * L + s];
                float acc1 = 0.f;
                int m = 0;
                for (; m + 1 < t; m += 2) {
                    acc0 = fmaf(lab[t * L + m], out[m * L + s], acc0);
                    acc1 = fmaf(lab[t * L + m + 1], out[(m + 1) * L + s], acc1);
                }
                if (m < t) acc0 = fmaf(lab[t * L + m], out[m * L + s], acc0);
                out[t * L + s] = acc0 + acc1;
            }
        }
        __syncthreads();
        {
            const int t = tid >> 2, q = tid & 3;
            const float *tsm = reinterpret_cast<const float *>(sm + TSM) + t * L + 8 * q;
            const float *psm = reinterpret_cast<const float *>(sm + PSM) + t * L + 8 * q;
            float xt[8], xp[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                xt[e] = tsm[e];
                xp[e] = psm[e];
            }
            store8_split(sm + T_HI, sm + T_LO, cm_off(t, 8 * q, L), xt);
            store8_split(sm + P_HI, sm + P_LO, cm_off(t, 8 * q, L), xp);
        }

        // ---- R2: W^T = A~^T T^T (lane 0), U~^T = V^T P^T (lane 16) ------------------
        issue_begin();
        if (tid == 0) {
            fence_after_sync();
            gemm_split(tmem + COL_Y, op_mn(sbase + GA_HI, sbase + GA_LO, 64), op_k(sbase + T_HI, sbase + T_LO, L),
                       idesc_bf16(64, 32, 1, 0), 2, false);
            gemm_split(tmem + COL_Y + (16u << 16), op_mn(sbase + VB, 0, 64), op_k(sbase + P_HI, sbase + P_LO, L),
                       idesc_bf16(64, 32, 1, 0), 2, false);
            commit(mbar);
        }
        if (!round_wait()) break;

        // ---- P2: stage W^T and U~^T as K-major A operands ------------------------------
        {
            float x[32];
            tmem_ld16(tmem + quad + COL_Y, *reinterpret_cast<float(*)[16]>(x));
            tmem_ld16(tmem + quad + COL_Y + 16, *reinterpret_cast<float(*)[16]>(x + 16));
            const int row = 16 * warp + (lane & 15);
            unsigned char *hi = sm + (lane < 16 ? WT_HI : UT_HI);
            unsigned char *lo = sm + (lane < 16 ? WT_LO : UT_LO);
#pragma unroll
            for (int q = 0; q < 4; ++q) store8_split(hi, lo, cm_off(row, 8 * q, L), x + 8 * q);
        }

        // ---- R3: M' = W^T B-, Q'^T = W^T L_rb^T, E, Y_loc^T -----------------------------
        issue_begin();
        if (tid == 0) {
            fence_after_sync();
            const Op wt = op_k(sbase + WT_HI, sbase + WT_LO, L);
            const Op ut = op_k(sbase + UT_HI, sbase + UT_LO, L);
            const Op vt = op_mn(sbase + VB, 0, 64);
            const Op bbar = op_mn(sbase + BBAR_HI, sbase + BBAR_LO, 64);
            const Op kbar = op_mn(sbase + KBAR_HI, sbase + KBAR_LO, 64);
            const Op lrb = op_k(sbase + LRB_HI, sbase + LRB_LO, L);
            const Op lrk = op_k(sbase + LRK_HI, sbase + LRK_LO, L);
            gemm_split(tmem + COL_X, wt, bbar, idesc_bf16(64, 64, 0, 1), 2, false);
            gemm_split(tmem + COL_X + 64, wt, lrb, idesc_bf16(64, 32, 0, 0), 2, false);
            gemm_split(tmem + COL_Z, ut, bbar, idesc_bf16(64, 64, 0, 1), 2, false);
            gemm_split(tmem + COL_Z, vt, kbar, idesc_bf16(64, 64, 1, 1), 2, true);
            gemm_split(tmem + COL_Z + 64, ut, lrb, idesc_bf16(64, 32, 0, 0), 2, false);
            gemm_split(tmem + COL_Z + 64, vt, lrk, idesc_bf16(64, 32, 1, 0), 2, true);
            commit(mbar);
        }
        if (!round_wait()) break;

        // ---- P3: M = diag(e^{c_31}) + M', Q^T = R~^T + Q'^T ---------------------------
        {
            float mrow[64], qrow[32];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tmem_ld16(tmem + quad + COL_X + 16 * q, *reinterpret_cast<float(*)[16]>(mrow + 16 * q));
            tmem_ld16(tmem + quad + COL_X + 64, *reinterpret_cast<float(*)[16]>(qrow));
            tmem_ld16(tmem + quad + COL_X + 80, *reinterpret_cast<float(*)[16]>(qrow + 16));
            if (lane < 16) {
                const int j = 16 * warp + lane;
                const float gam = reinterpret_cast<const float *>(sm + GAML)[j];
#pragma unroll
                for (int e = 0; e < 64; ++e) mrow[e] += (e == j) ? gam : 0.f;
#pragma unroll
                for (int t = 0; t < L; ++t) {
                    const uint32_t o = cm_off(L + t, j, 64);
                    qrow[t] += __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + GA_HI + o)) +
                               __bfloat162float(*reinterpret_cast<const __nv_bfloat16 *>(sm + GA_LO + o));
                }
#pragma unroll
                for (int q = 0; q < 8; ++q) store8_split(sm + M_HI, sm + M_LO, cm_off(j, 8 * q, 64), mrow + 8 * q);
#pragma unroll
                for (int q = 0; q < 4; ++q) store8_split(sm + Q_HI, sm + Q_LO, cm_off(j, 8 * q, L), qrow + 8 * q);
            }
        }

        // ---- R4: [S_out | Y^T] = [E | Y_loc^T] + S [M | Q^T] ----------------------------
        issue_begin();
        if (tid == 0) {
            fence_after_sync();
            const Op s = op_k(sbase + S_HI, sbase + S_LO, 64);
            gemm_split(tmem + COL_Z, s, op_mn(sbase + M_HI, sbase + M_LO, 64), idesc_bf16(64, 64, 0, 1), 4, true);
            gemm_split(tmem + COL_Z + 64, s, op_mn(sbase + Q_HI, sbase + Q_LO, L), idesc_bf16(64, 32, 0, 1), 4, true);
            commit(mbar);
        }
        if (!round_wait()) break;

        // ---- P4: y, next S operand, final state ------------------------------------------
        {
            float srow[64], yrow[32];
#pragma unroll
            for (int q = 0; q < 4; ++q)
                tmem_ld16(tmem + quad + COL_Z + 16 * q, *reinterpret_cast<float(*)[16]>(srow + 16 * q));
            tmem_ld16(tmem + quad + COL_Z + 64, *reinterpret_cast<float(*)[16]>(yrow));
            tmem_ld16(tmem + quad + COL_Z + 80, *reinterpret_cast<float(*)[16]>(yrow + 16));
            if (lane < 16) {
                const int i = 16 * warp + lane;
                OutT *yp = y + base + (size_t)t0 * tok_stride + i;
#pragma unroll
                for (int t = 0; t < L; ++t)
                    if (t < Lv) yp[(size_t)t * tok_stride] = from_f32<OutT>(yrow[t]);
#pragma unroll
                for (int q = 0; q < 8; ++q) store8_split(sm + S_HI, sm + S_LO, cm_off(i, 8 * q, 64), srow + 8 * q);
                if (c == nchunks - 1 && sT) {
#pragma unroll
                    for (int q = 0; q < 16; ++q)
                        store4(sT + st_base + (size_t)i * kN + 4 * q,
                               make_float4(srow[4 * q], srow[4 * q + 1], srow[4 * q + 2], srow[4 * q + 3]));
                }
            }
        }
        fence_smem_to_async();
        fence_before_sync();
    }

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
