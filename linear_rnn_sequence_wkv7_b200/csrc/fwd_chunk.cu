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
//   Gram^T = [b-; k-] [a'; r']^T                       (64 x 64; row s of b-
//            holds column s of L_ab and L_rb, row s of k- those of L_ak, L_rk)
//   L_ab, L_ak = strictly lower parts (t > s); L_rb, L_rk = lower parts (t >= s)
//   T = (I - L_ab)^{-1} (blocked: two 16x16 diagonal inverses by forward
//       substitution, then T21 = T22 L21 T11),  P = T L_ak      (CUDA cores, fp32)
//   W'^T = A'^T T^T,  U~^T = V^T P^T                   (u_t = S G w'_t + u~_t)
//   M = G (I + W'^T B-),  Q^T = G (R'^T + W'^T L_rb^T)   (G scales rows)
//   E = U~^T B- + V^T K-,  Y_loc^T = U~^T L_rb^T + V^T L_rk^T
//   S_out = S M + E,  Y^T = S Q^T + Y_loc^T          (state-dependent part)
//
// Precision: every tensor-core product uses bf16 hi/lo splits (x = hi + lo to
// 16 bits; three passes hi*hi + hi*lo + lo*hi, two when one side is an exact
// bf16 input such as v) with fp32 accumulation in TMEM.  A single tf32 or bf16
// pass is not accurate enough for the 2e-3 rms bound on this workload.
//
// Mapping: one CTA per (b, h), two CTAs per SM.  Warps 0-7 (256 threads)
// run the CUDA-core phases; warp 8 issues the tensor-core rounds.  Per chunk:
// P0 builds the decayed operands from the token tile (suffix products by
// warp shuffles); R1 Gram; P1 masks it and computes T and P; R2 W'^T, U~^T;
// P2 stages them; R3 M'', Q''^T, E, Y_loc^T; P3 finishes M and Q; R4
// accumulates the state product onto [E | Y_loc^T]; P4 writes y and stages
// S_out as the next chunk's operand.  Each round has a "ready" mbarrier (the
// 256 compute threads arrive after publishing their shared-memory writes) and
// a "done" mbarrier (tcgen05.commit); every wait is bounded.  The compute
// warps build chunk c+1's operands (P0) while R4 of chunk c runs, and R1 of
// chunk c+1 runs while they finish chunk c (P4).  Token tiles arrive by
// cp.async one chunk ahead.
//
// TMEM (256 columns).  An M=64 accumulator occupies lanes 16q..16q+15 of warp
// quadrant q; a second one at lane offset 16 fills lanes 16q+16..16q+31, so
// paired results are read by all 32 lanes of a warp:
//   X: cols [0, 96)     Gram (cols 0-63), then [M'' | Q''^T]
//   Y: cols [96, 128)   W'^T (lane 0) and U~^T (lane 16)
//   Z: cols [128, 224)  [E | Y_loc^T], then += S [M | Q^T] = [S_out | Y^T]
// L_rb and L_rk are stored next to b- and k- (one [64][96] operand), and M
// next to Q^T, so R3 and R4 run as N=96 products.
#include <algorithm>

#include "umma.cuh"

namespace wkv7 {

namespace chunk {

constexpr int L = 32;              // tokens per chunk
constexpr int NC = 256;            // compute threads (warps 0-7)
constexpr int NT = NC + 32;        // + the MMA warp
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_X = 0, COL_Y = 96, COL_Z = 128;
constexpr uint32_t LANE16 = 16u << 16;

// shared memory map (bytes)
constexpr uint32_t IN = 0;         // token tile: tensors w r k a b v, [32][128 B], 16-B chunks rotated by row
constexpr uint32_t IN_W = 0, IN_R = 4096, IN_K = 8192, IN_A = 12288, IN_B = 16384, IN_V = 20480;
constexpr uint32_t GA_HI = 24576, GA_LO = 32768;     // [64][64]: a' rows 0..31, r' rows 32..63
constexpr uint32_t BB_HI = 40960, BB_LO = 53248;     // [64][96]: rows s = [b-_s | L_rb[:, s]], rows 32+s = [k-_s | L_rk[:, s]]
constexpr uint32_t VB = 65536;                       // [32][64] exact bf16 v
constexpr uint32_t S_HI = 69632, S_LO = 77824;       // [64][64]
constexpr uint32_t R = 86016;                        // 24 KB, shared by short-lived buffers:
constexpr uint32_t T_HI = R, T_LO = R + 2048, P_HI = R + 4096, P_LO = R + 6144;    //   P1..R2: [32][32]
constexpr uint32_t ID32 = R;                         //   P2..R3: [32][32] bf16 identity
constexpr int LDT = 36;                              //   row pitch of L_ab^T (floats; bank spread)
constexpr uint32_t LABT = R + 8192;                  //   P1: fp32 L_ab^T [32][36]
constexpr uint32_t LAK = R + 12800;                  //   P1: fp32 L_ak [32][33] (padded)
constexpr uint32_t TSM = R + 17024;                  //   P1: fp32 T [32][32]
constexpr uint32_t ZSM = R + 21120;                  //   P1: fp32 [16][16]
constexpr uint32_t WT_HI = R + 8192, UT_HI = R + 12288, WT_LO = R + 16384, UT_LO = R + 20480;  // P2..R3: [64][32]
constexpr uint32_t MQ_HI = R, MQ_LO = R + 12288;     //   P3..R4: [64][96] = [M | Q^T]
constexpr uint32_t YSM = R;                          //   P4: fp32 [32][64]
constexpr uint32_t GAML = 110592;                    // fp32 [64]: G per channel
constexpr uint32_t BAR = 110848;                     // 8 mbarriers: ready R1..R4, done R1..R4
constexpr uint32_t TMEM_SLOT = 110912;
constexpr uint32_t FLAG = 110916;                    // set by whichever role gives up first
constexpr uint32_t CFLAG = 110920;                   // compute warps' copy, written by thread 0 only
constexpr uint32_t SMEM_BYTES = 110928;

constexpr long long kDrainCycles = 200000000LL;      // ~0.1 s to let committed tensor-core work finish
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

__device__ __forceinline__ void csync() { umma::named_sync(1, NC); }   // compute warps only

}  // namespace chunk

template <typename OutT>
__global__ void __launch_bounds__(chunk::NT, 2)
fwd_chunk_kernel(int T_total, int H, int t_seg, int nseg, const __nv_bfloat16 *__restrict__ r,
                 const __nv_bfloat16 *__restrict__ w, const __nv_bfloat16 *__restrict__ k,
                 const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ a,
                 const __nv_bfloat16 *__restrict__ b, const float *s0, long long s0_zstride, OutT *__restrict__ y,
                 float *sT, long long sT_zstride, int st_only_z, long long wait_limit) {
    using namespace chunk;
    using namespace umma;
    extern __shared__ __align__(1024) unsigned char sm[];
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, bb = blockIdx.y, z = blockIdx.z;
    // blockIdx.z selects a segment of the sequence; z >= nseg marks a
    // "transition" run of segment z - nseg (state starts at I, v taken as 0),
    // whose final state is the segment's linear map S -> S M_seg.
    const int seg = z % nseg;
    const bool transition = z >= nseg;
    const int t_begin = seg * t_seg;
    const int T = min(t_seg, T_total - t_begin);     // tokens of this segment
    const size_t tok_stride = (size_t)H * kN;
    const size_t base = (((size_t)bb * T_total + t_begin) * H + h) * kN;
    const size_t st_base = ((size_t)bb * H + h) * kN * kN;
    const float *s0p = s0 ? s0 + (size_t)z * s0_zstride + st_base : nullptr;
    float *sTp = (sT && (st_only_z < 0 || st_only_z == z)) ? sT + (st_only_z < 0 ? (size_t)z * sT_zstride : 0) + st_base
                                                            : nullptr;
    const int nchunks = (T + L - 1) / L;
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(sm + FLAG);
    volatile uint32_t *compute_flag = reinterpret_cast<volatile uint32_t *>(sm + CFLAG);
    int last_k = -1;                                 // issuer: last committed round and its parity
    uint32_t last_par = 0;
    auto ready_bar = [&](int k) { return sbase + BAR + 8u * (uint32_t)k; };        // k = 0..3 (R1..R4)
    auto done_bar = [&](int k) { return sbase + BAR + 32u + 8u * (uint32_t)k; };

    auto issue_tile = [&](int c) {        // compute threads only
        const __nv_bfloat16 *src[6] = {w, r, k, a, b, v};
        const int t0 = c * L;
        for (int x = tid; x < 6 * L * 8; x += NC) {
            const int ten = x >> 8, t = (x >> 3) & 31, ch = x & 7;
            if (t0 + t < T)
                cp_async16(sm + IN + ten * 4096 + in_off(t, ch), src[ten] + base + (size_t)(t0 + t) * tok_stride + ch * 8);
        }
        cp_async_commit();
    };

    // ---- set-up -------------------------------------------------------------------------
    if (tid == 0) {
        for (int kk = 0; kk < 4; ++kk) {
            mbar_init(ready_bar(kk), NC);
            mbar_init(done_bar(kk), 1);
        }
        *abort_flag = 0;
        *compute_flag = 0;
    }
    if (warp == 8) tmem_alloc(sbase + TMEM_SLOT, TMEM_COLS);
    if (tid < NC) {
        issue_tile(0);
        const int i = tid >> 2, c0 = (tid & 3) * 16;
#pragma unroll
        for (int g = 0; g < 2; ++g) {
            float x[8];
            if (transition) {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = (c0 + 8 * g + e == i) ? 1.f : 0.f;
            } else if (s0p) {
                const float4 u0 = load4(s0p + (size_t)i * kN + c0 + 8 * g);
                const float4 u1 = load4(s0p + (size_t)i * kN + c0 + 8 * g + 4);
                x[0] = u0.x; x[1] = u0.y; x[2] = u0.z; x[3] = u0.w; x[4] = u1.x; x[5] = u1.y; x[6] = u1.z; x[7] = u1.w;
            } else {
#pragma unroll
                for (int e = 0; e < 8; ++e) x[e] = 0.f;
            }
            store8_split(sm + S_HI, sm + S_LO, cm_off(i, c0 + 8 * g, 64), x);
        }
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + TMEM_SLOT);

    if (warp == 8) {
        // ================= MMA issuer =================
        if (lane == 0) {
            const uint32_t id_gram = idesc_bf16(64, 64, 0, 0), id_r2 = idesc_bf16(64, 32, 1, 0);
            const uint32_t id_km96 = idesc_bf16(64, 96, 0, 1), id_mm96 = idesc_bf16(64, 96, 1, 1);
            const OpD ga = opd_k(sbase + GA_HI, sbase + GA_LO, 64);
            const OpD bbk = opd_k(sbase + BB_HI, sbase + BB_LO, 96);           // [b-; k-] rows, K = cols 0..63
            const OpD at = opd_mn(sbase + GA_HI, sbase + GA_LO, 64);        // A'^T (rows 0..31 of GA)
            const OpD vt = opd_mn(sbase + VB, 0, 64);                          // V^T, exact
            const OpD tt = opd_k(sbase + T_HI, sbase + T_LO, L);
            const OpD pp = opd_k(sbase + P_HI, sbase + P_LO, L);
            const OpD wt = opd_k(sbase + WT_HI, sbase + WT_LO, L);
            const OpD ut = opd_k(sbase + UT_HI, sbase + UT_LO, L);
            const OpD bl = opd_mn(sbase + BB_HI, sbase + BB_LO, 96);          // [B- | L_rb^T]
            const OpD kl = opd_mn(sbase + BB_HI + 6144, sbase + BB_LO + 6144, 96);   // [K- | L_rk^T]
            const OpD ss = opd_k(sbase + S_HI, sbase + S_LO, 64);
            const OpD mq = opd_mn(sbase + MQ_HI, sbase + MQ_LO, 96);          // [M | Q^T]
            const OpD rt = opd_mn(sbase + GA_HI + 4096, sbase + GA_LO + 4096, 64);   // R'^T (rows 32..63 of GA)
            const OpD id = opd_k(sbase + ID32, 0, L);                          // identity, exact
            const uint32_t id_r = idesc_bf16(64, 32, 1, 0);
            for (int c = 0; c < nchunks; ++c) {
                const uint32_t par = (uint32_t)c & 1u;
                // R1: Gram
                if (!mbar_spin(ready_bar(0), par, wait_limit)) { *abort_flag = 1; break; }
                fence_after_sync();
                gemm_split_d(tmem + COL_X, bbk, ga, id_gram, 4, false);       // Gram^T
                commit(done_bar(0));
                last_k = 0;
                last_par = par;
                // R2: W'^T = A'^T T^T (lane 0), U~^T = V^T P^T (lane 16)
                if (!mbar_spin(ready_bar(1), par, wait_limit)) { *abort_flag = 1; break; }
                fence_after_sync();
                gemm_split_d(tmem + COL_Y, at, tt, id_r2, 2, false);
                gemm_split_d(tmem + COL_Y + LANE16, vt, pp, id_r2, 2, false);
                commit(done_bar(1));
                last_k = 1;
                last_par = par;
                // R3: [M'' | Q''^T] = W'^T [B- | L_rb^T];  [E | Y_loc^T] = U~^T [B- | L_rb^T] + V^T [K- | L_rk^T]
                if (!mbar_spin(ready_bar(2), par, wait_limit)) { *abort_flag = 1; break; }
                fence_after_sync();
                gemm_split_d(tmem + COL_X, wt, bl, id_km96, 2, false);
                gemm_split_d(tmem + COL_X + 64, rt, id, id_r, 2, true);       // Q''^T += R'^T
                gemm_split_d(tmem + COL_Z, ut, bl, id_km96, 2, false);
                gemm_split_d(tmem + COL_Z, vt, kl, id_mm96, 2, true);
                commit(done_bar(2));
                last_k = 2;
                last_par = par;
                // R4: [S_out | Y^T] += S [M | Q^T]
                if (!mbar_spin(ready_bar(3), par, wait_limit)) { *abort_flag = 1; break; }
                fence_after_sync();
                gemm_split_d(tmem + COL_Z, ss, mq, id_km96, 4, true);
                commit(done_bar(3));
                last_k = 3;
                last_par = par;
            }
        }
        __syncwarp();
    } else {
        // ================= compute warps =================
        const int q4 = warp & 3, hc = warp >> 2;     // TMEM lane quadrant, column half
        const uint32_t quad = (uint32_t)(32 * q4) << 16;
        const int sub = lane & 15;                   // row within the quadrant's 16
        const bool upper = lane >= 16;               // lanes reading the lane-16 accumulator

        // One lane polls, the others park at the barrier.  Only thread 0 reads
        // the shared abort flag (the issuer may set it at any time) and it
        // publishes its decision before the barrier, so all 256 threads take
        // the same branch afterwards.
        auto done_wait = [&](int kk, int c) -> bool {
            if (tid == 0) {
                const bool ok = mbar_spin(done_bar(kk), (uint32_t)c & 1u, wait_limit);
                if (!ok) *abort_flag = 1;
                *compute_flag = (!ok || *abort_flag) ? 1u : 0u;
            }
            csync();
            fence_after_sync();
            return *compute_flag == 0;
        };
        auto ready_arrive = [&](int kk) {
            fence_smem_to_async();
            fence_before_sync();
            mbar_arrive(ready_bar(kk));
        };

        auto P0 = [&](int Lv) {                   // decayed operands of one chunk
            const int g = warp, t = lane;         // channels 8g..8g+7, token t
            const bool valid = t < Lv;
            const uint32_t off = in_off(t, g);
            float wv[8], rv[8], kv[8], av[8], bv[8];
            bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + IN_W + off), wv);
            bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + IN_R + off), rv);
            bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + IN_K + off), kv);
            bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + IN_A + off), av);
            bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + IN_B + off), bv);
            const uint4 vraw = (valid && !transition) ? *reinterpret_cast<const uint4 *>(sm + IN_V + off)
                                                      : make_uint4(0, 0, 0, 0);
            float inc[8];
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
            float xa[8], xr[8], xb[8], xk[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) {
                const float n1 = __shfl_down_sync(0xffffffffu, inc[e], 1);
                const float nxt = lane == 31 ? 1.f : n1;
                const float G = __shfl_sync(0xffffffffu, inc[e], 0);
                if (lane == 0) {
                    reinterpret_cast<float *>(sm + GAML)[8 * g + e] = G;
                    if (G < kMinDecay) raise_status(WKV7_ERR_RANGE);
                }
                xa[e] = __fdividef(av[e], inc[e]);
                xr[e] = __fdividef(rv[e], nxt);
                xb[e] = bv[e] * nxt;
                xk[e] = kv[e] * nxt;
            }
            store8_split(sm + GA_HI, sm + GA_LO, cm_off(t, 8 * g, 64), xa);
            store8_split(sm + GA_HI, sm + GA_LO, cm_off(L + t, 8 * g, 64), xr);
            store8_split(sm + BB_HI, sm + BB_LO, cm_off(t, 8 * g, 96), xb);
            store8_split(sm + BB_HI, sm + BB_LO, cm_off(L + t, 8 * g, 96), xk);
            *reinterpret_cast<uint4 *>(sm + VB + cm_off(t, 8 * g, 64)) = vraw;
        };

        auto P1 = [&]() {                         // Gram -> L's; T = (I - L_ab)^{-1}; P = T L_ak
            {
                uint32_t r0[16], r1[16];
                tmem_ld16_nowait(tmem + quad + COL_X + 32 * hc, r0);
                tmem_ld16_nowait(tmem + quad + COL_X + 32 * hc + 16, r1);
                tmem_wait();
                if (!upper) {
                    const int rho = 16 * q4 + sub;
                    float g[32];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        g[e] = __uint_as_float(r0[e]);
                        g[16 + e] = __uint_as_float(r1[e]);
                    }
                    const int s = rho & 31;
                    if (rho < L && hc == 0) {         // column s of L_ab -> row s of L_ab^T
                        float *dst = reinterpret_cast<float *>(sm + LABT) + s * LDT;
#pragma unroll
                        for (int t4 = 0; t4 < 8; ++t4) {
                            float4 o;
                            o.x = 4 * t4 + 0 > s ? g[4 * t4 + 0] : 0.f;
                            o.y = 4 * t4 + 1 > s ? g[4 * t4 + 1] : 0.f;
                            o.z = 4 * t4 + 2 > s ? g[4 * t4 + 2] : 0.f;
                            o.w = 4 * t4 + 3 > s ? g[4 * t4 + 3] : 0.f;
                            *reinterpret_cast<float4 *>(dst + 4 * t4) = o;
                        }
                    } else if (rho >= L && hc == 0) { // column s of L_ak (rows padded to 33)
                        float *dst = reinterpret_cast<float *>(sm + LAK) + s;
#pragma unroll
                        for (int t = 0; t < L; ++t) dst[t * 33] = t > s ? g[t] : 0.f;
                    } else {                          // column s of L_rb / L_rk -> columns 64.. of row s / 32+s
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
                            float x[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e) x[e] = (8 * qq + e >= s) ? g[8 * qq + e] : 0.f;
                            store8_split(sm + BB_HI, sm + BB_LO, cm_off(rho, 64 + 8 * qq, 96), x);
                        }
                    }
                }
            }
            fence_before_sync();
            csync();
            const float *labt = reinterpret_cast<const float *>(sm + LABT);
            float *tsm = reinterpret_cast<float *>(sm + TSM);
            if (warp == 0) {                      // diagonal 16x16 blocks of T, one column per lane
                const int blk = lane >> 4, s = 16 * blk + sub;
                float acc[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) acc[e] = (e == sub) ? 1.f : 0.f;
#pragma unroll
                for (int m = 0; m < 15; ++m) {
                    const float x = acc[m];
                    const float *row = labt + (16 * blk + m) * LDT + 16 * blk;
#pragma unroll
                    for (int e4 = (m + 1) / 4; e4 < 4; ++e4) {
                        const float4 l4 = *reinterpret_cast<const float4 *>(row + 4 * e4);
                        const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                        for (int c4 = 0; c4 < 4; ++c4)
                            if (4 * e4 + c4 > m) acc[4 * e4 + c4] = fmaf(lv[c4], x, acc[4 * e4 + c4]);
                    }
                }
#pragma unroll
                for (int e = 0; e < 16; ++e) tsm[(16 * blk + e) * L + s] = acc[e];
            } else if (warp == 1) {               // upper-right block of T is zero
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int x = lane + 32 * e;
                    tsm[(x >> 4) * L + 16 + (x & 15)] = 0.f;
                }
            }
            csync();
            float *zsm = reinterpret_cast<float *>(sm + ZSM);
            {                                     // Z = L21 T11 (16 x 16), one entry per thread
                const int t = tid >> 4, s = tid & 15;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) acc = fmaf(labt[m * LDT + 16 + t], tsm[m * L + s], acc);
                zsm[t * 16 + s] = acc;
            }
            csync();
            {                                     // T21 = T22 Z
                const int t = tid >> 4, s = tid & 15;
                float acc = 0.f;
#pragma unroll
                for (int m = 0; m < 16; ++m) acc = fmaf(tsm[(16 + t) * L + 16 + m], zsm[m * 16 + s], acc);
                tsm[(16 + t) * L + s] = acc;
            }
            csync();
            {                                     // P = T L_ak and T, 4 rows per warp, one column per lane
                const float *lak = reinterpret_cast<const float *>(sm + LAK);
                const int s = lane;
                float pv[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m4 = 0; m4 < L / 4; ++m4) {
                    float4 tr[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i) tr[i] = *reinterpret_cast<const float4 *>(tsm + (4 * warp + i) * L + 4 * m4);
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const float lv = lak[(4 * m4 + c4) * 33 + s];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float tv = c4 == 0 ? tr[i].x : c4 == 1 ? tr[i].y : c4 == 2 ? tr[i].z : tr[i].w;
                            pv[i] = fmaf(tv, lv, pv[i]);
                        }
                    }
                }
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    const int t = 4 * warp + i;
                    const uint32_t o = cm_off(t, s, L);
                    const float tv = tsm[t * L + s];
                    __nv_bfloat16 hi = __float2bfloat16_rn(pv[i]);
                    *reinterpret_cast<__nv_bfloat16 *>(sm + P_HI + o) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(sm + P_LO + o) = __float2bfloat16_rn(pv[i] - __bfloat162float(hi));
                    hi = __float2bfloat16_rn(tv);
                    *reinterpret_cast<__nv_bfloat16 *>(sm + T_HI + o) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(sm + T_LO + o) = __float2bfloat16_rn(tv - __bfloat162float(hi));
                }
            }
        };

        auto P2 = [&]() {                         // stage W'^T (lanes 0-15) and U~^T (lanes 16-31)
            uint32_t r0[16];
            tmem_ld16_nowait(tmem + quad + COL_Y + 16 * hc, r0);
            tmem_wait();
            float x[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = __uint_as_float(r0[e]);
            const int row = 16 * q4 + sub;
            unsigned char *hi = sm + (upper ? UT_HI : WT_HI);
            unsigned char *lo = sm + (upper ? UT_LO : WT_LO);
            store8_split(hi, lo, cm_off(row, 16 * hc, L), x);
            store8_split(hi, lo, cm_off(row, 16 * hc + 8, L), x + 8);
            {   // identity operand for R3 (the T/P space is free once R2 is done)
                const int rr = tid >> 3, cc = 4 * (tid & 7);
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    *reinterpret_cast<__nv_bfloat16 *>(sm + ID32 + cm_off(rr, cc + e, L)) =
                        __float2bfloat16_rn(rr == cc + e ? 1.f : 0.f);
            }
        };

        auto P3 = [&]() {                         // [M | Q^T] rows j: M = G (I + M''), Q^T = G (R'^T + Q''^T) (R'^T added by R3)
            uint32_t r0[16], r1[16], r2[16];
            tmem_ld16_nowait(tmem + quad + COL_X + 48 * hc, r0);
            tmem_ld16_nowait(tmem + quad + COL_X + 48 * hc + 16, r1);
            tmem_ld16_nowait(tmem + quad + COL_X + 48 * hc + 32, r2);
            tmem_wait();
            if (!upper) {
                const int j = 16 * q4 + sub;
                const float G = reinterpret_cast<const float *>(sm + GAML)[j];
                float x[48];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    x[e] = __uint_as_float(r0[e]);
                    x[16 + e] = __uint_as_float(r1[e]);
                    x[32 + e] = __uint_as_float(r2[e]);
                }
#pragma unroll
                for (int e = 0; e < 48; ++e) {
                    const int col = 48 * hc + e;
                    x[e] = G * (x[e] + (col == j ? 1.f : 0.f));   // Q columns (col >= 64) never match j
                }
#pragma unroll
                for (int qq = 0; qq < 6; ++qq)
                    store8_split(sm + MQ_HI, sm + MQ_LO, cm_off(j, 48 * hc + 8 * qq, 96), x + 8 * qq);
            }
        };

        auto P4 = [&](int c, int Lv) {            // rows i of [S_out | Y^T]: next S operand, y, final state
            uint32_t r0[16], r1[16], r2[16];
            tmem_ld16_nowait(tmem + quad + COL_Z + 48 * hc, r0);
            tmem_ld16_nowait(tmem + quad + COL_Z + 48 * hc + 16, r1);
            tmem_ld16_nowait(tmem + quad + COL_Z + 48 * hc + 32, r2);
            tmem_wait();
            if (!upper) {
                const int i = 16 * q4 + sub;
                float x[48];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    x[e] = __uint_as_float(r0[e]);
                    x[16 + e] = __uint_as_float(r1[e]);
                    x[32 + e] = __uint_as_float(r2[e]);
                }
                const bool last = c == nchunks - 1 && sTp != nullptr;
                if (hc == 0) {                    // S columns 0..47
#pragma unroll
                    for (int qq = 0; qq < 6; ++qq) store8_split(sm + S_HI, sm + S_LO, cm_off(i, 8 * qq, 64), x + 8 * qq);
                    if (last) {
#pragma unroll
                        for (int qq = 0; qq < 12; ++qq)
                            store4(sTp + (size_t)i * kN + 4 * qq,
                                   make_float4(x[4 * qq], x[4 * qq + 1], x[4 * qq + 2], x[4 * qq + 3]));
                    }
                } else {                          // S columns 48..63, then y^T columns 0..31
#pragma unroll
                    for (int qq = 0; qq < 2; ++qq)
                        store8_split(sm + S_HI, sm + S_LO, cm_off(i, 48 + 8 * qq, 64), x + 8 * qq);
                    if (last) {
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq)
                            store4(sTp + (size_t)i * kN + 48 + 4 * qq,
                                   make_float4(x[4 * qq], x[4 * qq + 1], x[4 * qq + 2], x[4 * qq + 3]));
                    }
                    float *ysm = reinterpret_cast<float *>(sm + YSM);
#pragma unroll
                    for (int e = 0; e < L; ++e) ysm[e * kN + i] = x[16 + e];
                }
            }
            fence_before_sync();
            csync();
            if (y) {   // coalesced y rows: thread -> (token, 8 channels)
                const int t = tid >> 3, c8 = tid & 7;
                if (t < Lv) {
                    const float *ysm = reinterpret_cast<const float *>(sm + YSM) + t * kN + 8 * c8;
                    OutT *dst = y + base + (size_t)(c * L + t) * tok_stride + 8 * c8;
                    store4(dst, *reinterpret_cast<const float4 *>(ysm));
                    store4(dst + 4, *reinterpret_cast<const float4 *>(ysm + 4));
                }
            }
            csync();
        };

        // ---- compute schedule ----
        cp_async_wait<0>();
        csync();
        P0(min(L, T));
        csync();
        ready_arrive(0);                                   // R1(0)
        if (nchunks > 1) issue_tile(1);
        for (int c = 0; c < nchunks; ++c) {
            if (!done_wait(0, c)) break;                   // Gram(c)
            P1();
            ready_arrive(1);                               // R2(c)
            if (!done_wait(1, c)) break;
            P2();
            ready_arrive(2);                               // R3(c)
            if (!done_wait(2, c)) break;
            P3();
            ready_arrive(3);                               // R4(c)
            if (c + 1 < nchunks) {                         // next chunk's operands under R4(c)
                cp_async_wait<0>();
                csync();
                P0(min(L, T - (c + 1) * L));
                csync();
                ready_arrive(0);                           // R1(c+1), under P4(c)
                if (c + 2 < nchunks) issue_tile(c + 2);
            }
            if (!done_wait(3, c)) break;                   // R4(c)
            P4(c, min(L, T - c * L));
        }
        cp_async_wait<0>();
    }

    // ---- tear-down ----------------------------------------------------------------------
    __syncthreads();
    if (*abort_flag) {
        // a wait gave up: report it, let the tensor-core work already
        // committed finish (rounds complete in order, so the last commit
        // covers all), then release TMEM
        if (tid == 0) raise_status(WKV7_ERR_TIMEOUT);
        if (tid == NC && last_k >= 0) mbar_wait(done_bar(last_k), last_par, kDrainCycles);
        __syncthreads();
    }
    fence_after_sync();
    if (warp == 8) tmem_dealloc(tmem, TMEM_COLS);
}

// One launch of the chunked kernel over nz = gridDim.z segment runs.
static cudaError_t launch_chunk(int B, int T, int H, int t_seg, int nseg, int nz, wkv7_dtype y_dt, const void *r,
                                const void *w, const void *k, const void *v, const void *a, const void *b,
                                const float *s0, long long s0_zstride, void *y, float *sT, long long sT_zstride,
                                int st_only_z, long long wait_limit, cudaStream_t st) {
    dim3 grid(H, B, nz);
    const size_t smem = chunk::SMEM_BYTES;
#define WKV7_CHUNK_LAUNCH(O)                                                                                  \
    do {                                                                                                      \
        auto kern = fwd_chunk_kernel<O>;                                                                      \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);   \
        if (e != cudaSuccess) return e;                                                                       \
        kern<<<grid, chunk::NT, smem, st>>>(T, H, t_seg, nseg, (const __nv_bfloat16 *)r, (const __nv_bfloat16 *)w, \
                                            (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,               \
                                            (const __nv_bfloat16 *)a, (const __nv_bfloat16 *)b, s0, s0_zstride,   \
                                            (O *)y, sT, sT_zstride, st_only_z, wait_limit);                   \
    } while (0)
    if (y_dt == WKV7_F32) WKV7_CHUNK_LAUNCH(float);
    else WKV7_CHUNK_LAUNCH(__nv_bfloat16);
#undef WKV7_CHUNK_LAUNCH
    return cudaGetLastError();
}

// Segments combine: per head, S_in(0) = s0 (or 0) and
// S_in(k+1) = S_in(k) M_k + E_k, where E_k / M_k are the final states of the
// segment's plain and transition runs.  Writes S_in(k) for k < nseg.  One CTA
// (256 threads) per head, fp32 on the CUDA cores; thread -> row i, 16 columns.
__global__ void __launch_bounds__(256)
seg_combine_kernel(int BH, int nseg, const float *__restrict__ s0, const float *__restrict__ em,
                   float *__restrict__ sin_out) {
    __shared__ __align__(16) float Ssm[kN * kN];
    __shared__ __align__(16) float Msm[kN * kN];
    const int head = blockIdx.x, tid = threadIdx.x;
    const int i = tid >> 2, j0 = (tid & 3) * 16;
    const size_t hoff = (size_t)head * kN * kN;
    const size_t zstride = (size_t)BH * kN * kN;
    float cur[16];
#pragma unroll
    for (int e = 0; e < 16; ++e) cur[e] = s0 ? s0[hoff + (size_t)i * kN + j0 + e] : 0.f;
    for (int kk = 0; kk < nseg; ++kk) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            sin_out[(size_t)kk * zstride + hoff + (size_t)i * kN + j0 + e] = cur[e];
            Ssm[i * kN + j0 + e] = cur[e];
        }
        if (kk + 1 == nseg) break;
        const float *E = em + (size_t)kk * zstride + hoff;
        const float *M = em + (size_t)(nseg - 1 + kk) * zstride + hoff;
        for (int x = tid; x < kN * kN; x += 256) Msm[x] = M[x];
        __syncthreads();
        float acc[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[e] = E[(size_t)i * kN + j0 + e];
        for (int m = 0; m < kN; ++m) {
            const float sm_ = Ssm[i * kN + m];
#pragma unroll
            for (int e = 0; e < 16; ++e) acc[e] = fmaf(sm_, Msm[m * kN + j0 + e], acc[e]);
        }
        __syncthreads();
#pragma unroll
        for (int e = 0; e < 16; ++e) cur[e] = acc[e];
    }
}

// Relative time of one launch of n chunk CTAs that each run the same number
// of chunks, on sms SMs holding two CTAs each: a CTA alone on its SM runs at
// speed 1, two co-resident CTAs each take 1.46 times as long (measured on the
// prefill and long-context shapes); CTAs beyond the resident ones run in later
// rounds.
static double launch_rounds(long long n, int sms) {
    double t = 0.0;
    while (n > 0) {
        t += n > sms ? 1.46 : 1.0;
        n -= 2LL * sms;
    }
    return t;
}

// Number of sequence segments for a chunked forward over B*H heads.  The
// segmented form runs 2 (nseg - 1) summary runs and nseg output runs of T/nseg
// tokens each, i.e. about 3x the work of one pass, so it only pays when B*H
// CTAs leave most of the GPU idle.  Picks the nseg (segments of at least 4
// chunks) with the lowest estimated time, if that is below 95% of one pass;
// among near-ties (within 3%) the fewest segments, which need the least scratch.
int chunk_segments(int B, int T, int H, int sm_count) {
    static_assert(2 * chunk::SMEM_BYTES <= 228 * 1024, "two chunk CTAs per SM");
    const long long heads = (long long)B * H;
    const long long chunks = (T + chunk::L - 1) / chunk::L;
    if (sm_count <= 0 || heads <= 0) return 1;
    const long long max_n = std::min<long long>(64, chunks / 4);
    auto cost = [&](long long n) {
        return (launch_rounds(2 * (n - 1) * heads, sm_count) + launch_rounds(n * heads, sm_count)) / n;
    };
    double best = 0.95 * launch_rounds(heads, sm_count);
    for (long long n = 2; n <= max_n; ++n) best = std::min(best, cost(n));
    for (long long n = 2; n <= max_n; ++n)
        if (cost(n) <= 1.03 * best) return (int)n;
    return 1;
}

size_t chunk_workspace_bytes(int B, int T, int H, int nseg) {
    if (nseg <= 1) return 0;
    // E_k, M_k for segments 0..nseg-2 and S_in(k) for k < nseg
    return (size_t)(2 * (nseg - 1) + nseg) * B * H * kN * kN * sizeof(float);
}

cudaError_t fwd_chunk(int B, int T, int H, wkv7_dtype y_dt, const void *r, const void *w, const void *k,
                      const void *v, const void *a, const void *b, const float *s0, void *y, float *sT,
                      int nseg, void *workspace, long long wait_limit, cudaStream_t st) {
    if (nseg <= 1)
        return launch_chunk(B, T, H, T, 1, 1, y_dt, r, w, k, v, a, b, s0, 0, y, sT, 0, -1, wait_limit, st);
    const int chunks = (T + chunk::L - 1) / chunk::L;
    const int t_seg = ((chunks + nseg - 1) / nseg) * chunk::L;
    nseg = (T + t_seg - 1) / t_seg;
    const long long zst = (long long)B * H * kN * kN;
    float *em = static_cast<float *>(workspace);                // [2 (nseg-1)][B][H][64][64]
    float *sin = em + (size_t)2 * (nseg - 1) * zst;             // [nseg][B][H][64][64]
    // pass 1: E_k (s0 = 0) and M_k (s0 = I, v = 0) for segments 0..nseg-2, no y
    cudaError_t e = launch_chunk(B, T, H, t_seg, nseg - 1, 2 * (nseg - 1), y_dt, r, w, k, v, a, b, nullptr, 0,
                                 nullptr, em, zst, -1, wait_limit, st);
    if (e != cudaSuccess) return e;
    // pass 2: entry state of every segment
    seg_combine_kernel<<<B * H, 256, 0, st>>>(B * H, nseg, s0, em, sin);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
    // pass 3: every segment from its true entry state; the last one writes sT
    return launch_chunk(B, T, H, t_seg, nseg, nseg, y_dt, r, w, k, v, a, b, sin, zst, y, sT, 0, nseg - 1,
                        wait_limit, st);
}

}  // namespace wkv7
