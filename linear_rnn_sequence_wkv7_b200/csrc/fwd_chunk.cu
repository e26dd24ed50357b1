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
// The state-dependent products run transposed so that they are M=128 tensor-core
// products with one output row per TMEM lane:
//   [M''^T; Q''] = [B-^T; L_rb] W',   [E^T; Y_loc] = [B-^T; L_rb] U~ + [K-^T; L_rk] V
//   [S_out^T; Y] = [M^T; Q] S^T + [E^T; Y_loc]
// (96 rows used: 64 key rows j, then 32 tokens t).  W'^T and U~^T come from one
// stacked product [A'^T; V^T] [T^T | P^T] (the off-diagonal blocks are unused).
//
// Mapping: one CTA per (b, h), two CTAs per SM.  Warps 0-7 (256 threads) run
// the CUDA-core phases; warp 8 issues the tensor-core rounds.  Per chunk:
//   P0  decayed operands from the token tile (suffix products by shuffles)
//   R1  Gram^T = [b-; k-] [a'; r']^T                     (M=64, N=64)
//   P1  masks -> L's; T = (I - L_ab)^-1 and P = T L_ak on the CUDA cores
//   R2  [A'^T; V^T] [T^T | P^T] -> W'^T, U~^T             (M=128, N=64)
//   P2  stages [W' | U~] as the next B operand
//   R3  [M''^T; Q'' | E^T; Y_loc]                         (M=128, N=128 + 64)
//   P3  M^T = (I + M''^T) G, Q = (R' + Q'') G (G scales columns), written to
//       TMEM as the A operand of R4 (bf16 hi/lo pairs)
//   R4  += [M^T; Q] S^T, A from TMEM                      (M=128, N=64)
//   P4  S_out^T -> next S^T operand (and sT at the end); Y rows -> y directly
// Each round has a "ready" mbarrier (each compute warp arrives once its threads
// have published their writes) and a "done" mbarrier (tcgen05.commit); every
// wait is bounded.  P0 of chunk c+1 overlaps R4 of chunk c, R1 of chunk c+1
// overlaps P4 of chunk c.  Token tiles (w r k a b) arrive by cp.async one chunk
// ahead into a staging tile; v goes by cp.async straight into its operand.
//
// TMEM (256 columns):
//   X: cols [0, 64)     Gram^T (M=64 layout: lanes 16q..16q+15), then W'^T | U~^T
//   Z: cols [64, 192)   [M''^T; Q''] (0-63), [E^T; Y_loc] -> [S_out^T; Y] (64-127)
//   MQ: cols [192, 256) [M^T; Q] as bf16 pairs: hi 192-223, lo 224-255
#include <algorithm>

#include "umma.cuh"

namespace wkv7 {

namespace chunk {

constexpr int L = 32;              // tokens per chunk
constexpr int NC = 256;            // compute threads (warps 0-7)
constexpr int NT = NC + 32;        // + the MMA warp
constexpr uint32_t TMEM_COLS = 256;
constexpr uint32_t COL_X = 0, COL_Z = 64, COL_MQ = 192;
// dual runs: the second state's [S2_out^T; q] goes to [M''^T; Q'']'s columns
// (P3 has read them before R4 is issued); P4 parks S2_out in the [M^T; Q]
// columns until the next chunk's P3 turns it into the S2^T operand
constexpr uint32_t COL_S2 = COL_Z;

// shared memory map (bytes)
constexpr uint32_t IN_W = 0, IN_R = 4096, IN_K = 8192, IN_A = 12288, IN_B = 16384;   // [32][128 B], rotated
// [32 tokens][128]: a' (cols 0-63) | v (cols 64-127); R2's A and R1's B rows 0-31.
// RZ follows AV so that R1's B rows 32-63 are r'; RZ cols 64-127 are free space.
constexpr uint32_t AV_HI = 20480, RZ_HI = 28672, AV_LO = 36864, RZ_LO = 45056;
// [64][96]: rows s = [b-_s | L_rb[:, s]], rows 32+s = [k-_s | L_rk[:, s]]
constexpr uint32_t BB_HI = 53248, BB_LO = 65536;
constexpr uint32_t S_HI = 77824, S_LO = 86016;      // S^T [64 j][64 i]
constexpr uint32_t R = 94208;                       // short-lived buffers:
constexpr uint32_t TP_HI = R, TP_LO = R + 4096;     //   P1..R2: [64][32] = T rows 0-31, P rows 32-63
constexpr int LDT = 36;                             //   row pitch of L_ab^T (floats; bank spread)
constexpr uint32_t LABT = R + 8192;                 //   P1: fp32 L_ab^T [32][36]
constexpr uint32_t LAKT = R + 12800;                //   P1: fp32 L_ak^T [32][36]
constexpr uint32_t WU_HI = R, WU_LO = R + 8192;     //   P2..R3: [128][32] = W'^T rows, U~^T rows
constexpr uint32_t SMEM_BYTES = R + 17408;
// dual runs: S2^T operand [64 j][64 i], in the short-lived buffers: staged
// in P3 (R3 has read [W' | U~]), read by R4, overwritten by the next P1
constexpr uint32_t S2_HI = R, S2_LO = R + 8192;
static_assert(S2_LO + 8192 <= SMEM_BYTES, "S2^T fits in the short-lived buffers");
// in the free halves of RZ (bytes [1024, 2048) of each 2 KB group)
constexpr uint32_t TSM = RZ_HI + 1024;              // fp32 T, row t at TSM + (t/8)*2048 + (t%8)*128
constexpr uint32_t ZSM = RZ_LO + 1024;              // fp32 [16][16]
constexpr uint32_t GAML = RZ_LO + 3072;             // fp32 [64]: G per channel
constexpr uint32_t BAR = GAML + 256;                // 4 mbarriers: tcgen05.commit of R1..R4
constexpr uint32_t TMEM_SLOT = BAR + 64;
constexpr uint32_t FLAG = BAR + 68;                 // set by whichever role gives up first
// time-mix epilogue (EpiArgs): per-warp parts of the current-token weight
// u_t = sum_j r_t[j] rho[j] k_t[j], fp32 [32 t][8 warps]; and the two rounds of
// the per-head mean / variance exchange between the two halves of a y row
constexpr uint32_t UPART = RZ_LO + 5120;
constexpr uint32_t EXCH = RZ_LO + 7168;             // fp32 [2 rounds][2 halves][32 rows]
constexpr uint32_t GAMBET = RZ_LO + 7680;           // float2 [64]: (gamma, beta) of the head's channels
// the gate rows of the chunk, bf16 [32][64], arrive by cp.async in TSM's rows
// (free from the end of P1 to the next P1)
constexpr uint32_t BAR_EPI = 10;                    // named barrier of warps 2 and 6 (the y rows)
constexpr uint32_t BAR_T = 11;                      // named barrier of warps 0 and 1 (the inverse T)
constexpr uint32_t BAR_G = 12;                      // warps 0-1 have read the Gram; warps 4-7 may read theirs

constexpr long long kDrainCycles = 200000000LL;     // ~0.1 s to let committed tensor-core work finish
constexpr float kMinDecay = 1e-30f;                 // per-chunk decay floor (prod of 32 w)

__device__ __forceinline__ uint32_t in_off(int t, int ch) { return (uint32_t)(t * 128 + (((ch + t) & 7) << 4)); }
__device__ __forceinline__ uint32_t tsm_row(int t) { return TSM + (uint32_t)((t >> 3) * 2048 + (t & 7) * 128); }
__device__ __forceinline__ int hc_of(int warp) { return warp >> 2; }

__device__ __forceinline__ void bf8_to_f32(uint4 u, float *o) {
    const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        o[2 * q] = __uint_as_float(uu[q] << 16);
        o[2 * q + 1] = __uint_as_float(uu[q] & 0xffff0000u);
    }
}

__device__ __forceinline__ void csync() { umma::named_sync(1, NC); }   // compute warps only
// hand-off of round k (0..3 = R1..R4) between the compute warps and the issuer:
// named barriers over all NT threads
constexpr uint32_t BAR_READY = 2, BAR_DONE = 6;

}  // namespace chunk


// DUAL: a summary run that carries two states through the same chunk algebra,
// S from S_in (here 0, giving the segment's E) and S2 from I (giving M): the
// chunk's operands, T, W', M and Q do not depend on the state, so only the
// state round R4 and its read-out are done twice.  No y.  The second state
// needs no room of its own: R4 writes it into [M''^T; Q'']'s TMEM columns (P3
// has read them), P4 parks it in the [M^T; Q] columns (R4 has read them), and
// the next P3 turns it into its S2^T operand in the short-lived buffers (R3
// has read [W' | U~]).  So dual CTAs run two per SM, like the plain ones.
// EPI: the time-mix output epilogue (EpiArgs) replaces the y store.
// MQX: the checkpoint pass also exports every chunk's transition [M^T; Q] to mq.
template <typename OutT, bool DUAL, bool EPI, bool MQX = false>
__global__ void __launch_bounds__(chunk::NT, 2)
fwd_chunk_kernel(int T_total, int H, int t_seg, int nseg, const __nv_bfloat16 *__restrict__ r,
                 const __nv_bfloat16 *__restrict__ w, const __nv_bfloat16 *__restrict__ k,
                 const __nv_bfloat16 *__restrict__ v, const __nv_bfloat16 *__restrict__ a,
                 const __nv_bfloat16 *__restrict__ b, const float *s0, long long s0_zstride, OutT *__restrict__ y,
                 float *sT, long long sT_zstride, int st_only_z, long long wait_limit, float *ckpt,
                 float *m_out, long long m_zstride, int seg0, int first_out, EpiArgs epi, float *y0q,
                 uint4 *mq) {
    using namespace chunk;
    using namespace umma;
    extern __shared__ __align__(1024) unsigned char sm[];
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int h = blockIdx.x, bb = blockIdx.y, z = blockIdx.z;
    // blockIdx.z selects a segment of the sequence (seg0 + z, nseg of them
    // in this launch).
    const int seg = seg0 + z % nseg;
    const int t_begin = seg * t_seg;
    const int T = min(t_seg, T_total - t_begin);     // tokens of this segment
    const size_t tok_stride = (size_t)H * kN;
    const size_t base = (((size_t)bb * T_total + t_begin) * H + h) * kN;
    const size_t st_base = ((size_t)bb * H + h) * kN * kN;
    // A dual launch with first_out makes its first run an output run: from
    // s0, with y and checkpoints (its E is then the next segment's entry
    // state).  Every other dual run starts from 0 and writes no y.
    const bool out_run = !DUAL || (first_out && z == 0);
    const float *s0p = (s0 && out_run) ? s0 + (size_t)z * s0_zstride + st_base : nullptr;
    OutT *yo = out_run ? y : nullptr;
    float *sTp = (sT && (st_only_z < 0 || st_only_z == z)) ? sT + (st_only_z < 0 ? (size_t)z * sT_zstride : 0) + st_base
                                                            : nullptr;
    const int nchunks = (T + L - 1) / L;
    // optional state checkpoints: the state before every chunk of the whole
    // sequence, [B][H][ceil(T_total / L)][64][64]; a segment writes the slots
    // of its own chunks (t_seg is a multiple of L)
    float *ckp = (ckpt && out_run) ? ckpt + (((size_t)bb * H + h) * ((T_total + L - 1) / L) + t_begin / L) * kN * kN
                                   : nullptr;
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(sm + FLAG);
    int last_k = -1;                                 // issuer: last committed round and its parity
    uint32_t last_par = 0;
    auto done_bar = [&](int k) { return sbase + BAR + 8u * (uint32_t)k; };         // k = 0..3 (R1..R4)

    // token tile of chunk c (w r k a b) into the staging area; compute threads
    // only, thread -> (token, 16-byte chunk) of each tensor
    auto issue_in = [&](int c) {
        const int t = tid >> 3, ch = tid & 7;
        if (c < nchunks && c * L + t < T) {
            const size_t g = base + (size_t)(c * L + t) * tok_stride + ch * 8;
            const uint32_t o = in_off(t, ch);
            cp_async16(sm + IN_W + o, w + g);
            cp_async16(sm + IN_R + o, r + g);
            cp_async16(sm + IN_K + o, k + g);
            cp_async16(sm + IN_A + o, a + g);
            cp_async16(sm + IN_B + o, b + g);
        }
        cp_async_commit();
    };
    // v of chunk c straight into its operand (AV columns 64-127); rows past the
    // end keep the zeros P0 writes.  Transition runs keep v = 0.  The copies
    // are issued by warps 3 and 7, which have no rows in P3 (every compute
    // thread still commits a group, empty for the others).
    auto issue_v = [&](int c) {
        if (c < nchunks && (warp & 3) == 3) {
            const int t0 = c * L;
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                const int x = 32 * (warp >> 2) + lane + 64 * u;
                const int t = x >> 3, ch = x & 7;
                if (t0 + t < T)
                    cp_async16(sm + AV_HI + cm_off(t, 64 + 8 * ch, 128), v + base + (size_t)(t0 + t) * tok_stride + ch * 8);
            }
        }
        cp_async_commit();
    };

    // ---- set-up -------------------------------------------------------------------------
    if (tid == 0) {
        for (int kk = 0; kk < 4; ++kk) {
            mbar_init(done_bar(kk), 1);
        }
        *abort_flag = 0;
    }
    if (warp == 8) tmem_alloc(sbase + TMEM_SLOT, TMEM_COLS);
    if constexpr (EPI) {
        if (tid < kN)
            reinterpret_cast<float2 *>(sm + GAMBET)[tid] =
                make_float2(epi.gamma ? epi.gamma[(size_t)h * kN + tid] : 1.f,
                            epi.beta ? epi.beta[(size_t)h * kN + tid] : 0.f);
    }
    if (tid < NC) {
        {   // v columns of AV: lo always zero (v is exact)
            const int t = tid >> 3, ch = tid & 7;
            *reinterpret_cast<uint4 *>(sm + AV_LO + cm_off(t, 64 + 8 * ch, 128)) = make_uint4(0, 0, 0, 0);
        }
        issue_in(0);
        issue_v(0);
        // S^T operand: thread -> key column j of S, 16 value rows i
        const int j = tid & 63, part = tid >> 6;
        float x[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
            const int i = 16 * part + e;
            x[e] = s0p ? s0p[(size_t)i * kN + j] : 0.f;
        }
        store8_split(sm + S_HI, sm + S_LO, cm_off(j, 16 * part, 64), x);
        store8_split(sm + S_HI, sm + S_LO, cm_off(j, 16 * part + 8, 64), x + 8);
        if (ckp) {
#pragma unroll
            for (int e = 0; e < 16; ++e) ckp[(size_t)(16 * part + e) * kN + j] = x[e];
        }
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + TMEM_SLOT);

    if (warp == 8) {
        // ================= MMA issuer =================
        {
            const uint32_t id_gram = idesc_bf16(64, 64, 0, 0);
            const uint32_t id_r2 = idesc_bf16(128, 64, 1, 0);
            const uint32_t id_r3a = idesc_bf16(128, 128, 1, 0);
            const uint32_t id_r3b = idesc_bf16(128, 64, 1, 1);
            const uint32_t id_r4 = idesc_bf16(128, 64, 0, 1);
            const OpD bbk = opd_k(sbase + BB_HI, sbase + BB_LO, 96);          // [b-; k-] rows, K = cols 0..63
            const OpD avk = opd_k(sbase + AV_HI, sbase + AV_LO, 128);         // [a'; r'] rows, K = cols 0..63
            const OpD avm = opd_mn(sbase + AV_HI, sbase + AV_LO, 128);        // [A'^T; V^T], K = tokens
            const OpD tp = opd_k(sbase + TP_HI, sbase + TP_LO, L);            // [T; P] rows, K = tokens
            const OpD a1 = opd_mn(sbase + BB_HI, sbase + BB_LO, 96);          // [B-^T; L_rb], K = tokens
            const OpD a2 = opd_mn(sbase + BB_HI + 6144, sbase + BB_LO + 6144, 96);   // [K-^T; L_rk]
            const OpD wu = opd_k(sbase + WU_HI, sbase + WU_LO, L);            // [W' | U~], K = tokens
            const OpD vv = opd_mn(sbase + AV_HI + 1024, 0, 128);              // V, exact
            const OpD ss = opd_mn(sbase + S_HI, sbase + S_LO, 64);            // S^T, K = key j
            const OpD ss2 = opd_mn(sbase + S2_HI, sbase + S2_LO, 64);         // dual runs: S2^T
            // One tensor-core round: wait until the compute warps hand it over
            // (bar.arrive on its ready barrier), issue and commit it, wait for
            // the commit, and release the compute warps (bar.sync on its done
            // barrier).  The whole warp passes every barrier once per chunk
            // whatever happens; after a wait gives up nothing more is issued.
            auto round = [&](int rd, uint32_t par, auto &&issue) {
                named_sync(BAR_READY + rd, NT);
                fence_after_sync();
                if (lane == 0 && *abort_flag == 0u) {
                    issue();
                    commit(done_bar(rd));
                    last_k = rd;
                    last_par = par;
                    if (!mbar_spin_abortable(done_bar(rd), par, wait_limit, abort_flag)) *abort_flag = 1;
                }
                __syncwarp();
                fence_before_sync();
                named_arrive(BAR_DONE + rd, NT);
            };
            for (int c = 0; c < nchunks; ++c) {
                const uint32_t par = (uint32_t)c & 1u;
                round(0, par, [&] { gemm_split_d(tmem + COL_X, bbk, avk, id_gram, 4, false); });   // Gram^T
                round(1, par, [&] {                                                              // [W'^T; U~^T]
                    gemm_split_d(tmem + COL_X, avm, tp, id_r2, 2, false);
                });
                round(2, par, [&] {                         // [B-^T; L_rb] [W' | U~] + [K-^T; L_rk] [0 | V]
                    gemm_split_d(tmem + COL_Z, a1, wu, id_r3a, 2, false);
                    gemm_split_d(tmem + COL_Z + 64, a2, vv, id_r3b, 2, true);
                });
                round(3, par, [&] {                         // [S_out^T; Y] += [M^T; Q] S^T
                    gemm_split_ts(tmem + COL_Z + 64, tmem + COL_MQ, tmem + COL_MQ + 32, ss, id_r4, 4, true);
                    if constexpr (DUAL)                      // [S2_out^T; .] = [M^T; Q] S2^T (no E: v plays no part)
                        gemm_split_ts(tmem + COL_S2, tmem + COL_MQ, tmem + COL_MQ + 32, ss2, id_r4, 4, false);
                });
            }
        }
        __syncwarp();
    } else {
        // ================= compute warps =================
        const int q4 = warp & 3, hc = warp >> 2;     // TMEM lane quadrant, column half
        const uint32_t quad = (uint32_t)(32 * q4) << 16;
        const int sub = lane & 15;                   // row within the quadrant's 16 (M=64 layout)
        const bool upper = lane >= 16;
        const int rho = 32 * q4 + lane;              // row of an M=128 accumulator
        if constexpr (DUAL) {                        // the second state starts at I: S2^T rows, parked in
            if (q4 < 2) {                            // the [M^T; Q] columns until P3 of the first chunk
                uint32_t id0[16], id1[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    id0[e] = __float_as_uint(32 * hc + e == rho ? 1.f : 0.f);
                    id1[e] = __float_as_uint(32 * hc + 16 + e == rho ? 1.f : 0.f);
                }
                tmem_st16(tmem + quad + COL_MQ + 16 * hc, id0);          // the columns that this
                tmem_st16(tmem + quad + COL_MQ + 32 + 16 * hc, id1);     // warp's P3 overwrites
                tmem_st_wait();
            }
        }

        // Hand-offs with the issuer warp.  Waiting warps park at a hardware
        // barrier (no issue slots taken from the other CTA on the SM).  The
        // compute warps run one fixed schedule of barriers whatever happens;
        // after a wait gives up (abort flag, status word WKV7_ERR_TIMEOUT) the
        // remaining chunks run through on garbage so no warp is ever left at
        // a barrier.
        auto done_wait = [&](int kk, int) {
            named_sync(BAR_DONE + kk, NT);
            fence_after_sync();
        };
        // every thread publishes its own writes (shared memory to the async
        // proxy, TMEM stores) before it arrives
        auto ready_arrive = [&](int kk) {
            fence_smem_to_async();
            fence_before_sync();
            named_arrive(BAR_READY + kk, NT);
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
            if (Lv < L && !valid) {               // rows past the end of the sequence: no-op tokens, v = 0
#pragma unroll
                for (int e = 0; e < 8; ++e) { wv[e] = 1.f; rv[e] = 0.f; kv[e] = 0.f; av[e] = 0.f; bv[e] = 0.f; }
                *reinterpret_cast<uint4 *>(sm + AV_HI + cm_off(t, 64 + 8 * g, 128)) = make_uint4(0, 0, 0, 0);
            }
            float inc[8];
#pragma unroll
            for (int e = 0; e < 8; ++e) inc[e] = wv[e];
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
                xa[e] = __fdividef(av[e], inc[e]);
                xr[e] = __fdividef(rv[e], nxt);
                xb[e] = bv[e] * nxt;
                xk[e] = kv[e] * nxt;
            }
            if (lane == 0) {                      // G = p_0 of the warp's channels
                float4 *gp = reinterpret_cast<float4 *>(sm + GAML) + 2 * g;
                gp[0] = make_float4(inc[0], inc[1], inc[2], inc[3]);
                gp[1] = make_float4(inc[4], inc[5], inc[6], inc[7]);
                const float mn = fminf(fminf(fminf(inc[0], inc[1]), fminf(inc[2], inc[3])),
                                       fminf(fminf(inc[4], inc[5]), fminf(inc[6], inc[7])));
                if (mn < kMinDecay) raise_status(WKV7_ERR_RANGE);
            }
            if constexpr (EPI) {                  // part of u_t over this warp's 8 channels
                const float4 *rp = reinterpret_cast<const float4 *>(epi.rho + (size_t)h * kN + 8 * g);
                const float4 q0 = rp[0], q1 = rp[1];
                const float rr[8] = {q0.x, q0.y, q0.z, q0.w, q1.x, q1.y, q1.z, q1.w};
                float part = 0.f;
#pragma unroll
                for (int e = 0; e < 8; ++e) part = fmaf(rv[e] * rr[e], kv[e], part);
                reinterpret_cast<float *>(sm + UPART)[t * 8 + g] = part;
            }
            store8_split(sm + AV_HI, sm + AV_LO, cm_off(t, 8 * g, 128), xa);
            store8_split(sm + AV_HI, sm + AV_LO, cm_off(L + t, 8 * g, 128), xr);     // RZ rows
            store8_split(sm + BB_HI, sm + BB_LO, cm_off(t, 8 * g, 96), xb);
            store8_split(sm + BB_HI, sm + BB_LO, cm_off(L + t, 8 * g, 96), xk);
        };

        auto P1 = [&]() {                         // Gram -> L's; T = (I - L_ab)^{-1}; P = T L_ak
            {
                uint32_t r0[16], r1[16];
                if (warp >= 4) named_sync(BAR_G, 192);
                tmem_ld16_nowait(tmem + quad + COL_X + 32 * hc, r0);
                tmem_ld16_nowait(tmem + quad + COL_X + 32 * hc + 16, r1);
                tmem_wait();
                if (warp < 2) named_arrive(BAR_G, 192);
                if (!upper) {
                    const int row = 16 * q4 + sub;
                    float g[32];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        g[e] = __uint_as_float(r0[e]);
                        g[16 + e] = __uint_as_float(r1[e]);
                    }
                    const int s = row & 31;
                    if (hc == 0) {                    // column s of L_ab / L_ak -> row s of L_ab^T / L_ak^T
                        float *dst = reinterpret_cast<float *>(sm + (row < L ? LABT : LAKT)) + s * LDT;
#pragma unroll
                        for (int t4 = 0; t4 < 8; ++t4) {
                            float4 o;
                            o.x = 4 * t4 + 0 > s ? g[4 * t4 + 0] : 0.f;
                            o.y = 4 * t4 + 1 > s ? g[4 * t4 + 1] : 0.f;
                            o.z = 4 * t4 + 2 > s ? g[4 * t4 + 2] : 0.f;
                            o.w = 4 * t4 + 3 > s ? g[4 * t4 + 3] : 0.f;
                            *reinterpret_cast<float4 *>(dst + 4 * t4) = o;
                        }
                    } else {                          // column s of L_rb / L_rk -> columns 64.. of row s / 32+s
                        float u = 0.f;            // epilogue: u_s on the diagonal of L_rk
                        if (EPI && row >= L) {
                            const float4 *up = reinterpret_cast<const float4 *>(sm + UPART) + 2 * s;
                            const float4 u0 = up[0], u1 = up[1];
                            u = ((u0.x + u0.y) + (u0.z + u0.w)) + ((u1.x + u1.y) + (u1.z + u1.w));
                        }
#pragma unroll
                        for (int qq = 0; qq < 4; ++qq) {
                            float x[8];
#pragma unroll
                            for (int e = 0; e < 8; ++e)
                                x[e] = (8 * qq + e >= s) ? g[8 * qq + e] + (8 * qq + e == s ? u : 0.f) : 0.f;
                            store8_split(sm + BB_HI, sm + BB_LO, cm_off(row, 64 + 8 * qq, 96), x);
                        }
                    }
                }
            }
            const float *labt = reinterpret_cast<const float *>(sm + LABT);
            auto trow = [&](int t) { return reinterpret_cast<float *>(sm + tsm_row(t)); };
            if (warp < 2) {                       // diagonal 16x16 block 'warp' of T, one column per lane
                __syncwarp();                     // (its rows of L_ab^T are this warp's own)
                const int blk = warp, s = 16 * blk + sub;
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
                if (!upper) {
#pragma unroll
                    for (int e = 0; e < 16; ++e) trow(16 * blk + e)[s] = acc[e];
                }
            } else if (warp == 4) {               // upper-right block of T is zero
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const int x = lane + 32 * e;
                    trow(x >> 4)[16 + (x & 15)] = 0.f;
                }
            }
            float *zsm = reinterpret_cast<float *>(sm + ZSM);
            if (warp < 2) named_sync(BAR_T, 64);  // both diagonal blocks are in place
            if (tid < 64) {                       // Z = L21 T11 (16 x 16), four entries of a row per thread
                const int t = tid >> 2, s0 = 4 * (tid & 3);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m = 0; m < 16; ++m) {
                    const float l = labt[m * LDT + 16 + t];
                    const float4 tv = *reinterpret_cast<const float4 *>(trow(m) + s0);
                    acc[0] = fmaf(l, tv.x, acc[0]);
                    acc[1] = fmaf(l, tv.y, acc[1]);
                    acc[2] = fmaf(l, tv.z, acc[2]);
                    acc[3] = fmaf(l, tv.w, acc[3]);
                }
                *reinterpret_cast<float4 *>(zsm + t * 16 + s0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
                named_sync(BAR_T, 64);
            }
            if (tid < 64) {                       // T21 = T22 Z
                const int t = tid >> 2, s0 = 4 * (tid & 3);
                float acc[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
                    const float4 a4 = *reinterpret_cast<const float4 *>(trow(16 + t) + 16 + 4 * m4);
                    const float av[4] = {a4.x, a4.y, a4.z, a4.w};
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        const float4 zv = *reinterpret_cast<const float4 *>(zsm + (4 * m4 + c4) * 16 + s0);
                        acc[0] = fmaf(av[c4], zv.x, acc[0]);
                        acc[1] = fmaf(av[c4], zv.y, acc[1]);
                        acc[2] = fmaf(av[c4], zv.z, acc[2]);
                        acc[3] = fmaf(av[c4], zv.w, acc[3]);
                    }
                }
                *reinterpret_cast<float4 *>(trow(16 + t) + s0) = make_float4(acc[0], acc[1], acc[2], acc[3]);
            }
            fence_before_sync();
            csync();                              // T, L_ak (warps 2-3) and the zero block are in place
            {   // P = T L_ak, skipping the zero 16x16 blocks: P11 = T11 L11,
                // P21 = T21 L11 + T22 L21, P22 = T22 L22, P12 = 0.  Half-warp
                // kk (0..15), lane column s: row kk (cols < 16, m < 16), row
                // 16 + kk (cols < 16, all m; cols >= 16, m >= 16).
                const float *lakt = reinterpret_cast<const float *>(sm + LAKT);
                const int kk = 2 * warp + (lane >> 4), s = lane & 15;
                const float *ta = trow(kk), *tb = trow(16 + kk);
                const float *la = lakt + s * LDT, *lc = lakt + (16 + s) * LDT;   // columns s, 16 + s of L_ak
                float pa = 0.f, pb = 0.f, pc = 0.f;
#pragma unroll
                for (int m4 = 0; m4 < 4; ++m4) {
                    const float4 xa = *reinterpret_cast<const float4 *>(ta + 4 * m4);
                    const float4 xb = *reinterpret_cast<const float4 *>(tb + 4 * m4);
                    const float4 l4 = *reinterpret_cast<const float4 *>(la + 4 * m4);
                    const float va[4] = {xa.x, xa.y, xa.z, xa.w}, vb[4] = {xb.x, xb.y, xb.z, xb.w};
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w};
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        pa = fmaf(va[c4], lv[c4], pa);
                        pb = fmaf(vb[c4], lv[c4], pb);
                    }
                }
#pragma unroll
                for (int m4 = 4; m4 < 8; ++m4) {
                    const float4 xb = *reinterpret_cast<const float4 *>(tb + 4 * m4);
                    const float4 l4 = *reinterpret_cast<const float4 *>(la + 4 * m4);
                    const float4 c4v = *reinterpret_cast<const float4 *>(lc + 4 * m4);
                    const float vb[4] = {xb.x, xb.y, xb.z, xb.w};
                    const float lv[4] = {l4.x, l4.y, l4.z, l4.w}, cv[4] = {c4v.x, c4v.y, c4v.z, c4v.w};
#pragma unroll
                    for (int c4 = 0; c4 < 4; ++c4) {
                        pb = fmaf(vb[c4], lv[c4], pb);
                        pc = fmaf(vb[c4], cv[c4], pc);
                    }
                }
                auto put = [&](uint32_t hi_base, uint32_t lo_base, int row, int col, float x) {
                    const __nv_bfloat16 hi = __float2bfloat16_rn(x);
                    const uint32_t o = cm_off(row, col, L);
                    *reinterpret_cast<__nv_bfloat16 *>(sm + hi_base + o) = hi;
                    *reinterpret_cast<__nv_bfloat16 *>(sm + lo_base + o) = __float2bfloat16_rn(x - __bfloat162float(hi));
                };
                put(TP_HI, TP_LO, kk, s, ta[s]);
                put(TP_HI, TP_LO, kk, 16 + s, ta[16 + s]);
                put(TP_HI, TP_LO, 16 + kk, s, tb[s]);
                put(TP_HI, TP_LO, 16 + kk, 16 + s, tb[16 + s]);
                put(TP_HI, TP_LO, L + kk, s, pa);
                put(TP_HI, TP_LO, L + kk, 16 + s, 0.f);
                put(TP_HI, TP_LO, L + 16 + kk, s, pb);
                put(TP_HI, TP_LO, L + 16 + kk, 16 + s, pc);
            }
        };

        auto P2 = [&]() {                         // rows of W'^T (quadrants 0-1) and U~^T (2-3) -> [W' | U~]
            uint32_t r0[16];
            const uint32_t col = (q4 < 2 ? 0u : 32u) + 16u * (uint32_t)hc;
            tmem_ld16_nowait(tmem + quad + COL_X + col, r0);
            tmem_wait();
            float x[16];
#pragma unroll
            for (int e = 0; e < 16; ++e) x[e] = __uint_as_float(r0[e]);
            store8_split(sm + WU_HI, sm + WU_LO, cm_off(rho, 16 * hc, L), x);
            store8_split(sm + WU_HI, sm + WU_LO, cm_off(rho, 16 * hc + 8, L), x + 8);
        };

        auto P3 = [&](int c) {                    // rows of [M^T; Q] -> TMEM A operand of R4
            if (q4 == 3) return;
            if constexpr (DUAL) {                 // S2^T row rho (parked by the last P4) -> its operand
                if (q4 < 2) {
                    uint32_t s0[16], s1[16];
                    tmem_ld16_nowait(tmem + quad + COL_MQ + 16 * hc, s0);
                    tmem_ld16_nowait(tmem + quad + COL_MQ + 32 + 16 * hc, s1);
                    tmem_wait();
                    float x2[32];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        x2[e] = __uint_as_float(s0[e]);
                        x2[16 + e] = __uint_as_float(s1[e]);
                    }
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        store8_split(sm + S2_HI, sm + S2_LO, cm_off(rho, 32 * hc + 8 * u, 64), x2 + 8 * u);
                }
            }
            uint32_t r0[16], r1[16];
            tmem_ld16_nowait(tmem + quad + COL_Z + 32 * hc, r0);
            tmem_ld16_nowait(tmem + quad + COL_Z + 32 * hc + 16, r1);
            float gv[32];
            const float4 *g4 = reinterpret_cast<const float4 *>(sm + GAML) + 8 * hc;
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const float4 q = g4[u];
                gv[4 * u] = q.x; gv[4 * u + 1] = q.y; gv[4 * u + 2] = q.z; gv[4 * u + 3] = q.w;
            }
            float add[32];
            if (q4 < 2) {                         // M^T row j' = rho: + identity
#pragma unroll
                for (int e = 0; e < 32; ++e) add[e] = (32 * hc + e == rho) ? 1.f : 0.f;
            } else {                              // Q row t: + r'_t (hi + lo)
                const int t = rho - 64;
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    float hv[8], lv[8];
                    bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + AV_HI + cm_off(L + t, 32 * hc + 8 * u, 128)), hv);
                    bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + AV_LO + cm_off(L + t, 32 * hc + 8 * u, 128)), lv);
#pragma unroll
                    for (int e = 0; e < 8; ++e) add[8 * u + e] = hv[e] + lv[e];
                }
            }
            tmem_wait();
            float xv[32];
#pragma unroll
            for (int e = 0; e < 16; e += 2) {     // packed pairs: (acc + add) * G
                const float2 lo = __fmul2_rn(make_float2(gv[e], gv[e + 1]),
                                             __fadd2_rn(make_float2(__uint_as_float(r0[e]), __uint_as_float(r0[e + 1])),
                                                        make_float2(add[e], add[e + 1])));
                const float2 hi = __fmul2_rn(make_float2(gv[16 + e], gv[17 + e]),
                                             __fadd2_rn(make_float2(__uint_as_float(r1[e]), __uint_as_float(r1[e + 1])),
                                                        make_float2(add[16 + e], add[17 + e])));
                xv[e] = lo.x; xv[e + 1] = lo.y; xv[16 + e] = hi.x; xv[17 + e] = hi.y;
            }
            uint32_t ph[16], pl[16];
#pragma unroll
            for (int e2 = 0; e2 < 16; ++e2) {
                const float x0 = xv[2 * e2], x1 = xv[2 * e2 + 1];
                const __nv_bfloat162 hp = __floats2bfloat162_rn(x0, x1);
                const uint32_t hu = *reinterpret_cast<const uint32_t *>(&hp);
                const float2 rr = __ffma2_rn(make_float2(__uint_as_float(hu << 16), __uint_as_float(hu & 0xffff0000u)),
                                             make_float2(-1.f, -1.f), make_float2(x0, x1));
                const __nv_bfloat162 lp = __floats2bfloat162_rn(rr.x, rr.y);
                ph[e2] = hu;
                pl[e2] = *reinterpret_cast<const uint32_t *>(&lp);
            }
            tmem_st16(tmem + quad + COL_MQ + 16 * hc, ph);
            tmem_st16(tmem + quad + COL_MQ + 32 + 16 * hc, pl);
            if (MQX && out_run) {
                // optional chunk transitions, written with the checkpoints: the
                // same hi / lo pairs as row rho of chunk c's image (kMqChunkVec
                // 16-byte words per chunk, indexed like ckpt); the address is
                // formed here from the launch parameters so that it holds no
                // register over the rest of the chunk
                uint4 *dst = mq + ((((size_t)blockIdx.y * H + blockIdx.x) * ((T_total + L - 1) / L) +
                                    (size_t)(seg0 + blockIdx.z % nseg) * (t_seg / L) + c) *
                                   kMqChunkVec);
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const uint32_t o = cm_off(rho, 32 * hc + 8 * u, kN) >> 4;
                    dst[o] = make_uint4(ph[4 * u], ph[4 * u + 1], ph[4 * u + 2], ph[4 * u + 3]);
                    dst[kMqChunkVec / 2 + o] = make_uint4(pl[4 * u], pl[4 * u + 1], pl[4 * u + 2], pl[4 * u + 3]);
                }
            }
            tmem_st_wait();
        };

        auto P4 = [&](int c, int Lv) {            // rows of [S_out^T; Y]
            if (q4 == 3) return;
            uint32_t r0[16], r1[16];
            tmem_ld16_nowait(tmem + quad + COL_Z + 64 + 32 * hc, r0);
            tmem_ld16_nowait(tmem + quad + COL_Z + 64 + 32 * hc + 16, r1);
            tmem_wait();
            float x[32];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                x[e] = __uint_as_float(r0[e]);
                x[16 + e] = __uint_as_float(r1[e]);
            }
            if (q4 < 2) {                         // column j = rho of S_out, rows i = 32 hc + e
#pragma unroll
                for (int u = 0; u < 4; ++u)
                    store8_split(sm + S_HI, sm + S_LO, cm_off(rho, 32 * hc + 8 * u, 64), x + 8 * u);
                if (c == nchunks - 1 && sTp != nullptr) {
#pragma unroll
                    for (int e = 0; e < 32; ++e) sTp[(size_t)(32 * hc + e) * kN + rho] = x[e];
                }
                if (ckp != nullptr && c + 1 < nchunks) {
                    float *dst = ckp + (size_t)(c + 1) * kN * kN + rho;
#pragma unroll
                    for (int e = 0; e < 32; ++e) dst[(size_t)(32 * hc + e) * kN] = x[e];
                }
                if constexpr (DUAL) {             // the second state: parked in the [M^T; Q] columns
                    tmem_ld16_nowait(tmem + quad + COL_S2 + 32 * hc, r0);
                    tmem_ld16_nowait(tmem + quad + COL_S2 + 32 * hc + 16, r1);
                    tmem_wait();
                    // R4 has read [M^T; Q]; the parked row goes to the columns that
                    // this warp's next P3 reads it from and then overwrites (its hi
                    // and lo words), so no other warp's P3 store can land on it first
                    tmem_st16(tmem + quad + COL_MQ + 16 * hc, r0);
                    tmem_st16(tmem + quad + COL_MQ + 32 + 16 * hc, r1);
                    if (c == nchunks - 1 && m_out != nullptr) {
                        float *mp = m_out + (size_t)z * m_zstride + st_base;
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            mp[(size_t)(32 * hc + e) * kN + rho] = __uint_as_float(r0[e]);
                            mp[(size_t)(32 * hc + 16 + e) * kN + rho] = __uint_as_float(r1[e]);
                        }
                    }
                    tmem_st_wait();
                }
            } else if (DUAL && !yo && y0q != nullptr) {
                // a summary run's y rows: y0 (its output from S = 0) and q = M_{<=t} r_t
                // (the second state's rows, from I), fp32 [2][B][T][H][64] at the
                // tokens' own positions; y_t = y0_t + S_in q_t once S_in is known
                const int t = rho - 64;
                if (t < Lv) {
                    const size_t off = base + (size_t)(c * L + t) * tok_stride + 32 * hc;
                    float4 *d0 = reinterpret_cast<float4 *>(y0q + off);
#pragma unroll
                    for (int u = 0; u < 8; ++u) d0[u] = make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]);
                }
                tmem_ld16_nowait(tmem + quad + COL_S2 + 32 * hc, r0);
                tmem_ld16_nowait(tmem + quad + COL_S2 + 32 * hc + 16, r1);
                tmem_wait();
                if (t < Lv) {
                    const size_t off = base + (size_t)(c * L + t) * tok_stride + 32 * hc;
                    const size_t plane = (size_t)gridDim.y * T_total * H * kN;
                    float4 *d1 = reinterpret_cast<float4 *>(y0q + plane + off);
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        d1[u] = make_float4(__uint_as_float(r0[4 * u]), __uint_as_float(r0[4 * u + 1]),
                                            __uint_as_float(r0[4 * u + 2]), __uint_as_float(r0[4 * u + 3]));
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        d1[4 + u] = make_float4(__uint_as_float(r1[4 * u]), __uint_as_float(r1[4 * u + 1]),
                                                __uint_as_float(r1[4 * u + 2]), __uint_as_float(r1[4 * u + 3]));
                }
            } else if (EPI && yo) {               // epilogue: z row t from o row t (halves in warps 2, 6)
                const int t = rho - 64;
                float *ex = reinterpret_cast<float *>(sm + EXCH);
                float s1 = 0.f;
#pragma unroll
                for (int e = 0; e < 32; ++e) s1 += x[e];
                ex[32 * hc + lane] = s1;
                named_sync(BAR_EPI, 64);
                const float mu = (s1 + ex[32 * (1 - hc) + lane]) * (1.f / kN);
                float s2 = 0.f;
#pragma unroll
                for (int e = 0; e < 32; ++e) s2 = fmaf(x[e] - mu, x[e] - mu, s2);
                ex[64 + 32 * hc + lane] = s2;
                named_sync(BAR_EPI, 64);
                const float inv = rsqrtf((s2 + ex[64 + 32 * (1 - hc) + lane]) * (1.f / kN) + epi.eps);
                if (t < Lv) {
                    OutT *dst = yo + base + (size_t)(c * L + t) * tok_stride + 32 * hc;
                    const float4 *gb = reinterpret_cast<const float4 *>(sm + GAMBET) + 16 * hc;
#pragma unroll
                    for (int u = 0; u < 4; ++u) {  // 8 channels at a time
                        float gv[8];
                        if (epi.g) bf8_to_f32(*reinterpret_cast<const uint4 *>(sm + tsm_row(t) + 64 * hc + 16 * u), gv);
                        else for (int e = 0; e < 8; ++e) gv[e] = 1.f;
                        float zz[8];
#pragma unroll
                        for (int e2 = 0; e2 < 4; ++e2) {   // (gamma, beta) pairs of two channels
                            const float4 p = gb[4 * u + e2];
                            const int e = 2 * e2;
                            zz[e] = fmaf((x[8 * u + e] - mu) * inv, p.x, p.y) * gv[e];
                            zz[e + 1] = fmaf((x[8 * u + e + 1] - mu) * inv, p.z, p.w) * gv[e + 1];
                        }
                        store4(dst + 8 * u, make_float4(zz[0], zz[1], zz[2], zz[3]));
                        store4(dst + 8 * u + 4, make_float4(zz[4], zz[5], zz[6], zz[7]));
                    }
                }
            } else if (yo) {                      // y row t, channels 32 hc .. 32 hc + 31
                const int t = rho - 64;
                if (t < Lv) {
                    OutT *dst = yo + base + (size_t)(c * L + t) * tok_stride + 32 * hc;
#pragma unroll
                    for (int u = 0; u < 8; ++u)
                        store4(dst + 4 * u, make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]));
                }
            }
        };

        // ---- compute schedule ----
        // cp.async groups are committed in a fixed order: [w r k a b](c+1)
        // while R2(c) runs (the warps wait for it anyway; Gram(c) done means
        // every warp has finished P0(c), so the staging tile is free), [v](c+1)
        // at the start of P3(c) (both possibly empty).
        cp_async_wait<0>();
        csync();
        P0(min(L, T));
        ready_arrive(0);                                   // R1(0)
        for (int c = 0; c < nchunks; ++c) {
            done_wait(0, c);                               // Gram(c)
            P1();
            cp_async_wait<0>();                            // v(c) is in place
            ready_arrive(1);                               // R2(c)
            issue_in(c + 1);                               // under R2(c)
            done_wait(1, c);
            if constexpr (EPI) {                           // gate rows of chunk c (P1's T rows are dead)
                if (yo && epi.g && warp % 4 == 2) {
                    const int t = lane;
                    if (c * L + t < T) {
                        const __nv_bfloat16 *src = static_cast<const __nv_bfloat16 *>(epi.g) + base +
                                                   (size_t)(c * L + t) * tok_stride + 32 * hc_of(warp);
#pragma unroll
                        for (int q = 0; q < 4; ++q) cp_async16(sm + tsm_row(t) + 64 * hc_of(warp) + 16 * q, src + 8 * q);
                    }
                }
                cp_async_commit();                         // (empty for the other threads)
            }
            P2();
            ready_arrive(2);                               // R3(c)
            done_wait(2, c);
            issue_v(c + 1);                                // v(c) is no longer read
            P3(c);
            ready_arrive(3);                               // R4(c)
            if (c + 1 < nchunks) {                         // next chunk's operands under R4(c)
                cp_async_wait<1>();                        // tile c+1 is in place
                csync();                                   // ... for all threads; P3(c) reads are done
                P0(min(L, T - (c + 1) * L));
                ready_arrive(0);                           // R1(c+1), under P4(c)
            }
            done_wait(3, c);                               // R4(c)
            if constexpr (EPI) cp_async_wait<1>();         // the gate of chunk c (all but v(c+1))
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
                                int st_only_z, long long wait_limit, cudaStream_t st, float *ckpt = nullptr,
                                int seg0 = 0, EpiArgs epi = EpiArgs{}, uint4 *mq = nullptr) {
    dim3 grid(H, B, nz);
    const size_t smem = chunk::SMEM_BYTES;
#define WKV7_CHUNK_LAUNCH(O, E, X)                                                                            \
    do {                                                                                                      \
        auto kern = fwd_chunk_kernel<O, false, E, X>;                                                         \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);   \
        if (e != cudaSuccess) return e;                                                                       \
        kern<<<grid, chunk::NT, smem, st>>>(T, H, t_seg, nseg, (const __nv_bfloat16 *)r, (const __nv_bfloat16 *)w, \
                                            (const __nv_bfloat16 *)k, (const __nv_bfloat16 *)v,               \
                                            (const __nv_bfloat16 *)a, (const __nv_bfloat16 *)b, s0, s0_zstride,   \
                                            (O *)y, sT, sT_zstride, st_only_z, wait_limit, ckpt, nullptr, 0,  \
                                            seg0, 0, epi, nullptr, mq);                                       \
    } while (0)
    if (mq) {                                     // checkpoints with the transitions (no epilogue)
        if (epi.rho) return cudaErrorInvalidValue;
        if (y && y_dt == WKV7_F32) WKV7_CHUNK_LAUNCH(float, false, true);
        else WKV7_CHUNK_LAUNCH(__nv_bfloat16, false, true);
    } else if (epi.rho) {
        if (y_dt == WKV7_F32) WKV7_CHUNK_LAUNCH(float, true, false);
        else WKV7_CHUNK_LAUNCH(__nv_bfloat16, true, false);
    } else {
        if (y_dt == WKV7_F32) WKV7_CHUNK_LAUNCH(float, false, false);
        else WKV7_CHUNK_LAUNCH(__nv_bfloat16, false, false);
    }
#undef WKV7_CHUNK_LAUNCH
    return cudaGetLastError();
}

// One launch of dual summary runs over nz segments of t_seg tokens: E of
// segment z (its final state from 0) to e_out + z e_zstride, M (from I, v read
// as 0) to m_out + z m_zstride.  With y or ckpt given, the first segment
// instead runs from s0 and writes them: its "E" is its true final state.
static cudaError_t launch_dual(int B, int T, int H, int t_seg, int nz, const void *r, const void *w, const void *k,
                               const void *v, const void *a, const void *b, float *e_out, long long e_zstride,
                               float *m_out, long long m_zstride, long long wait_limit, cudaStream_t st,
                               void *y = nullptr, wkv7_dtype y_dt = WKV7_F32, const float *s0 = nullptr,
                               float *ckpt = nullptr, EpiArgs epi = EpiArgs{}, float *y0q = nullptr,
                               uint4 *mq = nullptr) {

    dim3 grid(H, B, nz);
    const size_t smem = chunk::SMEM_BYTES;
    const int first_out = (y != nullptr || ckpt != nullptr) ? 1 : 0;
    using bf = __nv_bfloat16;
#define WKV7_DUAL_LAUNCH(O, E, X)                                                                              \
    do {                                                                                                       \
        auto kern = fwd_chunk_kernel<O, true, E, X>;                                                           \
        cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);    \
        if (e != cudaSuccess) return e;                                                                        \
        kern<<<grid, chunk::NT, smem, st>>>(T, H, t_seg, nz, (const bf *)r, (const bf *)w, (const bf *)k,      \
                                            (const bf *)v, (const bf *)a, (const bf *)b, s0, 0, (O *)y, e_out, \
                                            e_zstride, -1, wait_limit, ckpt, m_out, m_zstride, 0, first_out,   \
                                            epi, y0q, mq);                                                     \
    } while (0)
    if (mq) {                                     // segmented checkpoints with the transitions
        if (epi.rho) return cudaErrorInvalidValue;
        if (y && y_dt == WKV7_F32) WKV7_DUAL_LAUNCH(float, false, true);
        else WKV7_DUAL_LAUNCH(bf, false, true);
    } else if (epi.rho && first_out) {
        if (y_dt == WKV7_BF16) WKV7_DUAL_LAUNCH(bf, true, false);
        else WKV7_DUAL_LAUNCH(float, true, false);
    } else {
        if (y_dt == WKV7_BF16) WKV7_DUAL_LAUNCH(bf, false, false);
        else WKV7_DUAL_LAUNCH(float, false, false);
    }
#undef WKV7_DUAL_LAUNCH
    return cudaGetLastError();
}

// Chain of affine state maps, per head: X_0 = s0 (I when s0_eye, zeros when
// s0 is null), X_{k+1} = X_k M_k + E_k for k < nsteps (X_k M_k^T + E_k with
// transpose_m), with M_k at m_base + k m_stride and E_k at e_base + k e_stride
// ([B*H][64][64] each; strides may be negative; E read as zeros when e_base
// is null).  With out_stride != 0 writes every X_k,
// k <= nsteps, at out + k out_stride; else only X_nsteps at out.  The rows of
// X are independent: CTA (head, rb) owns rows 8 rb .. 8 rb + 7, thread ->
// (row, two columns); M_k is staged in shared memory.  fp32 on CUDA cores.
constexpr int kCombineRows = 8;

__global__ void __launch_bounds__(256)
seg_combine_kernel(int nsteps, const float *__restrict__ s0, int s0_eye, const float *__restrict__ e_base,
                   long long e_stride, const float *__restrict__ m_base, long long m_stride,
                   float *__restrict__ out, long long out_stride, int transpose_m) {
    __shared__ __align__(16) float Msm[kN * kN];
    __shared__ float Ssm[kCombineRows][kN];
    const int head = blockIdx.x, tid = threadIdx.x;
    const int rr = tid >> 5, c2 = 2 * (tid & 31);
    const int i = kCombineRows * blockIdx.y + rr;
    const size_t hoff = (size_t)head * kN * kN, eoff = hoff + (size_t)i * kN + c2;
    float2 cur = s0 ? *reinterpret_cast<const float2 *>(s0 + eoff)
                    : (s0_eye ? make_float2(i == c2 ? 1.f : 0.f, i == c2 + 1 ? 1.f : 0.f) : make_float2(0.f, 0.f));
    for (int kk = 0;; ++kk) {
        if (out_stride != 0 || kk == nsteps) *reinterpret_cast<float2 *>(out + kk * out_stride + eoff) = cur;
        if (kk == nsteps) break;
        const float *M = m_base + kk * m_stride + hoff;
        Ssm[rr][c2] = cur.x;
        Ssm[rr][c2 + 1] = cur.y;
        if (transpose_m) {                            // Msm[m][c] = M[c][m]
            for (int x = tid; x < kN * kN; x += 256) Msm[(x & 63) * kN + (x >> 6)] = M[x];
        } else {
            for (int x = tid; x < kN * kN / 4; x += 256)
                reinterpret_cast<float4 *>(Msm)[x] = reinterpret_cast<const float4 *>(M)[x];
        }
        __syncthreads();
        float2 acc = e_base ? *reinterpret_cast<const float2 *>(e_base + kk * e_stride + eoff) : make_float2(0.f, 0.f);
#pragma unroll 16
        for (int m = 0; m < kN; ++m) {
            const float sv = Ssm[rr][m];
            const float2 mv = *reinterpret_cast<const float2 *>(Msm + m * kN + c2);
            acc.x = fmaf(sv, mv.x, acc.x);
            acc.y = fmaf(sv, mv.y, acc.y);
        }
        __syncthreads();
        cur = acc;
    }
}

// The output of segments seg_first..nseg-1 from their summary runs: a segment's state
// at token t is S_in M_{<=t} + E_{<=t}, so y_t = y0_t + S_in q_t, with y0_t
// its output from S = 0 and q_t = M_{<=t} r_t the second state's output
// (both fp32 in y0q = [2][B][T][H][64]).  One CTA of 128 threads per (head,
// segment, 256 tokens of it): S_in of the segment staged transposed in shared
// memory once, then 64-token tiles of q.  Thread -> 4 tokens x 8 value rows
// (4 rg .. 4 rg + 3 and 32 + 4 rg .. 32 + 4 rg + 3, so a quarter-warp reads 128
// contiguous bytes of S_in and one broadcast q): 6 shared loads per 16 packed
// fp32 FMAs.
constexpr int kFixTokens = 256, kFixTile = 64;

template <typename OutT>
__global__ void __launch_bounds__(128)
seg_fixup_kernel(int T, int H, int t_seg, int seg_first, const float *__restrict__ y0q,
                 const float *__restrict__ sin, long long sin_zstride, OutT *__restrict__ y) {
    __shared__ __align__(16) float St[kN][kN + 4];    // St[i][i'] = S_in[i'][i]
    __shared__ __align__(16) float Qs[kFixTile][kN + 4];
    const int head = blockIdx.x, seg = blockIdx.y + seg_first, tid = threadIdx.x;
    const int bb = head / H, h = head % H;
    const int t_lo = seg * t_seg + kFixTokens * blockIdx.z;
    const int t_hi = min(T, min((seg + 1) * t_seg, t_lo + kFixTokens));
    if (t_lo >= t_hi) return;
    const float *S = sin + (size_t)(seg - seg_first) * sin_zstride + (size_t)head * kN * kN;
    for (int x = tid; x < kN * kN; x += 128) St[x & 63][x >> 6] = S[x];
    const size_t tok_stride = (size_t)H * kN, plane = (size_t)gridDim.x / H * T * tok_stride;
    const size_t base = ((size_t)bb * T * H + h) * kN;
    const int tg = tid >> 3, rg = tid & 7;
    for (int t0 = t_lo; t0 < t_hi; t0 += kFixTile) {
        const int nt = min(kFixTile, t_hi - t0);
        __syncthreads();                              // St staged / the previous tile's Qs consumed
        for (int x = tid; x < kFixTile * kN / 4; x += 128) {
            const int r = x / (kN / 4), c4 = x % (kN / 4);
            *reinterpret_cast<float4 *>(&Qs[r][4 * c4]) =
                r < nt ? *reinterpret_cast<const float4 *>(y0q + plane + base + (size_t)(t0 + r) * tok_stride + 4 * c4)
                       : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncthreads();
        float2 acc[4][4];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = 4 * tg + k;
            float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
            if (r < nt) {
                const float *src = y0q + base + (size_t)(t0 + r) * tok_stride;
                a = *reinterpret_cast<const float4 *>(src + 4 * rg);
                b = *reinterpret_cast<const float4 *>(src + 32 + 4 * rg);
            }
            acc[k][0] = make_float2(a.x, a.y); acc[k][1] = make_float2(a.z, a.w);
            acc[k][2] = make_float2(b.x, b.y); acc[k][3] = make_float2(b.z, b.w);
        }
#pragma unroll 8
        for (int i = 0; i < kN; ++i) {
            const float4 s0 = *reinterpret_cast<const float4 *>(&St[i][4 * rg]);
            const float4 s1 = *reinterpret_cast<const float4 *>(&St[i][32 + 4 * rg]);
            const float2 p0 = make_float2(s0.x, s0.y), p1 = make_float2(s0.z, s0.w);
            const float2 p2 = make_float2(s1.x, s1.y), p3 = make_float2(s1.z, s1.w);
#pragma unroll
            for (int k = 0; k < 4; ++k) {
                const float qv = Qs[4 * tg + k][i];
                const float2 q2 = make_float2(qv, qv);
                acc[k][0] = __ffma2_rn(q2, p0, acc[k][0]);
                acc[k][1] = __ffma2_rn(q2, p1, acc[k][1]);
                acc[k][2] = __ffma2_rn(q2, p2, acc[k][2]);
                acc[k][3] = __ffma2_rn(q2, p3, acc[k][3]);
            }
        }
#pragma unroll
        for (int k = 0; k < 4; ++k) {
            const int r = 4 * tg + k;
            if (r < nt) {
                OutT *dst = y + base + (size_t)(t0 + r) * tok_stride;
                store4(dst + 4 * rg, make_float4(acc[k][0].x, acc[k][0].y, acc[k][1].x, acc[k][1].y));
                store4(dst + 32 + 4 * rg, make_float4(acc[k][2].x, acc[k][2].y, acc[k][3].x, acc[k][3].y));
            }
        }
    }
}

// Fix-up of segments seg_first .. nseg - 1, segment k taking its entry state
// from sin + (k - seg_first) sin_zstride.
static cudaError_t launch_fixup(int B, int T, int H, int t_seg, int seg_first, int nseg, wkv7_dtype y_dt,
                                const float *y0q, const float *sin, long long sin_zstride, void *y, cudaStream_t st) {
    if (nseg <= seg_first) return cudaSuccess;
    const dim3 grid(B * H, nseg - seg_first, (t_seg + kFixTokens - 1) / kFixTokens);
    if (y_dt == WKV7_F32)
        seg_fixup_kernel<float>
            <<<grid, 128, 0, st>>>(T, H, t_seg, seg_first, y0q, sin, sin_zstride, static_cast<float *>(y));
    else
        seg_fixup_kernel<__nv_bfloat16>
            <<<grid, 128, 0, st>>>(T, H, t_seg, seg_first, y0q, sin, sin_zstride, static_cast<__nv_bfloat16 *>(y));
    return cudaGetLastError();
}

static cudaError_t launch_combine(int B, int H, int nsteps, const float *s0, bool s0_eye, const float *e_base,
                                  long long e_stride, const float *m_base, long long m_stride, float *out,
                                  long long out_stride, cudaStream_t st, bool transpose_m = false) {
    seg_combine_kernel<<<dim3(B * H, kN / kCombineRows), 256, 0, st>>>(nsteps, s0, s0_eye ? 1 : 0, e_base, e_stride,
                                                                       m_base, m_stride, out, out_stride,
                                                                       transpose_m ? 1 : 0);
    return cudaGetLastError();
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

// Relative time of one launch of n dual summary runs: they fit two per SM
// like the plain runs, each chunk step about kDualCost times a plain one at
// the same co-residency (measured on the long-context shape: 8.64 vs 7.66 us
// per chunk step with two CTAs per SM).
constexpr double kDualCost = 1.13;
static double dual_rounds(long long n, int sms) {
    return n > 0 ? kDualCost * launch_rounds(n, sms) : 0.0;
}

// Number of sequence segments for a chunked forward over B*H heads.  The
// segmented form runs nseg - 1 dual summary runs (the first of them also the
// output run of segment 0) and nseg - 1 output runs of T/nseg tokens each,
// about twice the work of one pass, so it only pays when B*H CTAs leave most
// of the GPU idle.  Picks the nseg (segments of at least 4
// chunks) with the lowest estimated time, if that is below 95% of one pass;
// among near-ties (within 3%) the fewest segments, which need the least scratch.
// With summarize_last (the summary / continue pair) the last segment's summary
// runs too and one segment means two launches (summary, then output), so the
// cost model counts nseg summary runs and n = 1 competes on equal terms.
int chunk_segments(int B, int T, int H, int sm_count, bool summarize_last) {
    static_assert(2 * (chunk::SMEM_BYTES + 1024) <= 228 * 1024, "two chunk CTAs per SM");
    const long long heads = (long long)B * H;
    const long long chunks = (T + chunk::L - 1) / chunk::L;
    if (sm_count <= 0 || heads <= 0) return 1;
    const long long max_n = std::min<long long>(64, chunks / 4);
    // plain forward: dual runs for segments 0..n-2 (the first also writes its
    // y), output runs for segments 1..n-1; summary / continue: both for all n
    const long long extra = summarize_last ? 0 : 1;
    auto cost = [&](long long n) {
        return (dual_rounds((n - extra) * heads, sm_count) + launch_rounds((n - extra) * heads, sm_count)) / n;
    };
    double best = summarize_last ? cost(1) : 0.95 * launch_rounds(heads, sm_count);
    for (long long n = 2; n <= max_n; ++n) best = std::min(best, cost(n));
    for (long long n = 2; n <= max_n; ++n)
        if (cost(n) <= 1.03 * best) return (int)n;
    return 1;
}

// Segment length (whole chunks) and the number of non-empty segments for a
// request of nseg segments over T tokens.
static void seg_split(int T, int nseg, int &t_seg, int &n) {
    const int chunks = (T + chunk::L - 1) / chunk::L;
    t_seg = ((chunks + nseg - 1) / nseg) * chunk::L;
    n = (T + t_seg - 1) / t_seg;
}

// Fix-up form of the segmented forward (no checkpoints, no epilogue): one
// dual launch over all nseg segments, the first an output run from s0 and the
// others keeping their y0 and q rows; a chain for the entry states; the
// fix-up y = y0 + S_in q.  Cost in units of one CTA alone running all of T:
// nseg dual runs of T/nseg tokens, plus the fix-up pass, which moves 640 B
// per head-token (measured ~1.6e-10 s per head-token against ~4.9 us per
// chunk of one CTA alone: 1.0e-3 units per head).
constexpr double kFixupPerHead = 1.0e-3;
int chunk_segments_fixup(int B, int T, int H, int sm_count) {
    const long long heads = (long long)B * H;
    const long long chunks = (T + chunk::L - 1) / chunk::L;
    if (sm_count <= 0 || heads <= 0) return 1;
    const long long max_n = std::min<long long>(64, chunks / 4);
    auto cost = [&](long long n) {
        const long long per = (chunks + n - 1) / n;
        return dual_rounds(n * heads, sm_count) * (double)per / (double)chunks + kFixupPerHead * (double)heads;
    };
    double best = 0.95 * launch_rounds(heads, sm_count);
    for (long long n = 2; n <= max_n; ++n) best = std::min(best, cost(n));
    for (long long n = 2; n <= max_n; ++n)
        if (cost(n) <= 1.03 * best) return (int)n;
    return 1;
}

size_t chunk_fixup_workspace_bytes(int B, int T, int H, int nseg) {
    if (nseg <= 1) return 0;
    // E_k, M_k and S_in(k + 1) for every segment, then y0 and q for every token
    return (size_t)3 * nseg * B * H * kN * kN * sizeof(float) + (size_t)2 * B * T * H * kN * sizeof(float);
}

size_t chunk_workspace_bytes(int B, int T, int H, int nseg) {
    if (nseg <= 1) return 0;
    // E_k, M_k for segments 0..nseg-2 and S_in(k) for k < nseg
    return (size_t)(2 * (nseg - 1) + nseg) * B * H * kN * kN * sizeof(float);
}

size_t summary_workspace_bytes(int B, int T, int H, int nseg) {
    if (nseg <= 1) return 0;
    // E_k, M_k for every segment, the entry states and the final state, then
    // y0 and q of every token for the continue's fix-up
    return (size_t)(3 * nseg + 1) * B * H * kN * kN * sizeof(float) + (size_t)2 * B * T * H * kN * sizeof(float);
}

// The summary of an empty sequence: E = 0, M = I (one thread per element of both).
__global__ void summary_empty_kernel(long long zst, float *summary) {
    const long long x = (long long)blockIdx.x * blockDim.x + threadIdx.x;
    if (x >= 2 * zst) return;
    const int e = (int)(x % (kN * kN));
    summary[x] = (x >= zst && e / kN == e % kN) ? 1.f : 0.f;
}

// Affine summary of a whole sequence, S_out = S_in M + E, E to summary[0] and
// M to summary[1] ([B][H][64][64] each).  One segment: one dual run (E from
// S_in = 0 and M from S_in = I with v read as 0).  nseg segments: a dual run
// for every segment in one launch (their summaries stay in the workspace for
// fwd_chunk_continue), then E and M of the whole sequence by chaining them:
// E from 0 through every (E_k, M_k), M from I through the M_k.
cudaError_t fwd_chunk_summary(int B, int T, int H, const void *r, const void *w, const void *k, const void *v,
                              const void *a, const void *b, float *summary, int nseg, void *workspace,
                              long long wait_limit, cudaStream_t st) {
    const long long zst = (long long)B * H * kN * kN;
    if (T == 0) {
        summary_empty_kernel<<<(unsigned)((2 * zst + 255) / 256), 256, 0, st>>>(zst, summary);
        return cudaGetLastError();
    }
    if (nseg <= 1) return launch_dual(B, T, H, T, 1, r, w, k, v, a, b, summary, zst, summary + zst, zst, wait_limit, st);
    int t_seg, n;
    seg_split(T, nseg, t_seg, n);
    float *em = static_cast<float *>(workspace);                // E_0..E_{n-1}, M_0..M_{n-1}
    float *y0q = em + (3 * n + 1) * zst;                         // y0, q of every token (for the continue)
    cudaError_t e = launch_dual(B, T, H, t_seg, n, r, w, k, v, a, b, em, zst, em + n * zst, zst, wait_limit, st,
                                nullptr, WKV7_F32, nullptr, nullptr, EpiArgs{}, y0q);
    if (e != cudaSuccess) return e;
    e = launch_combine(B, H, n, nullptr, false, em, zst, em + n * zst, zst, summary, 0, st);
    if (e != cudaSuccess) return e;
    return launch_combine(B, H, n, nullptr, true, nullptr, 0, em + n * zst, zst, summary + zst, 0, st);
}

// The forward of a sequence from its entry state s_in after fwd_chunk_summary
// ran on the same inputs, segment count and workspace: the entry state of
// every segment from the kept (E_k, M_k), then every segment's output run.
cudaError_t fwd_chunk_continue(int B, int T, int H, wkv7_dtype y_dt, const void *r, const void *w, const void *k,
                               const void *v, const void *a, const void *b, const float *s_in, void *y, float *sT,
                               int nseg, void *workspace, long long wait_limit, cudaStream_t st) {
    if (nseg <= 1)
        return launch_chunk(B, T, H, T, 1, 1, y_dt, r, w, k, v, a, b, s_in, 0, y, sT, 0, -1, wait_limit, st);
    const long long zst = (long long)B * H * kN * kN;
    int t_seg, n;
    seg_split(T, nseg, t_seg, n);
    float *em = static_cast<float *>(workspace);
    float *sin = em + 2 * n * zst;                  // entry states of segments 0 .. n - 1, then the final state
    const float *y0q = em + (3 * n + 1) * zst;      // kept by the summary
    cudaError_t e = launch_combine(B, H, n, s_in, false, em, zst, em + n * zst, zst, sin, zst, st);
    if (e != cudaSuccess) return e;
    // every segment in fix-up form: y = y0 + S_in q (the summary's dual runs
    // started every segment from 0 and from I)
    e = launch_fixup(B, T, H, t_seg, 0, n, y_dt, y0q, sin, zst, y, st);
    if (e != cudaSuccess || sT == nullptr) return e;
    return cudaMemcpyAsync(sT, sin + n * zst, zst * sizeof(float), cudaMemcpyDeviceToDevice, st);
}

// dL/dS before each of nseg consecutive segments, last segment first:
// adj[nseg] = dsT (or 0), adj[k] = adj[k+1] M_k^T + F_k, with M_k in
// summary[k] = [E_k; M_k] and F_k the segment's own state gradient.
cudaError_t compose_adjoints(int B, int H, int nseg, const float *dsT, const float *summary, const float *F,
                             float *adj, cudaStream_t st) {
    const long long zst = (long long)B * H * kN * kN;
    if (nseg == 0) return launch_combine(B, H, 0, dsT, false, nullptr, 0, nullptr, 0, adj, 0, st);
    return launch_combine(B, H, nseg, dsT, false, F + (nseg - 1) * zst, -zst, summary + (2LL * (nseg - 1) + 1) * zst,
                          -2 * zst, adj + nseg * zst, -zst, st, true);
}

// Entry states of nseg consecutive segments and the state after the last:
// out[0] = s0 (or 0), out[k+1] = out[k] M_k + E_k, with summary[k] = [E_k; M_k].
cudaError_t compose_states(int B, int H, int nseg, const float *s0, const float *summary, float *out,
                           cudaStream_t st) {
    const long long zst = (long long)B * H * kN * kN;
    const float *m0 = summary ? summary + zst : nullptr;     // nseg = 0 reads no summary
    return launch_combine(B, H, nseg, s0, false, summary, 2 * zst, m0, 2 * zst, out, zst, st);
}

// The forward in the fix-up form over nseg segments (see chunk_segments_fixup).
static cudaError_t fwd_chunk_fixup(int B, int T, int H, wkv7_dtype y_dt, const void *r, const void *w,
                                   const void *k, const void *v, const void *a, const void *b, const float *s0,
                                   void *y, float *sT, int nseg, void *workspace, long long wait_limit,
                                   cudaStream_t st) {
    int t_seg;
    seg_split(T, nseg, t_seg, nseg);
    if (nseg <= 1)
        return launch_chunk(B, T, H, T, 1, 1, y_dt, r, w, k, v, a, b, s0, 0, y, sT, 0, -1, wait_limit, st);
    const long long zst = (long long)B * H * kN * kN;
    float *em = static_cast<float *>(workspace);        // E_k [nseg], then M_k [nseg]
    float *sin = em + 2 * nseg * zst;                    // S_in(1) .. S_in(nseg) (the last = final state)
    float *y0q = sin + nseg * zst;                       // [2][B][T][H][64]
    // pass 1: segment 0 from s0 writes y (its "E" is S_in(1)); segments >= 1
    // from 0 and from I keep E_k, M_k and their y0, q rows
    cudaError_t e = launch_dual(B, T, H, t_seg, nseg, r, w, k, v, a, b, em, zst, em + nseg * zst, zst, wait_limit,
                                st, y, y_dt, s0, nullptr, EpiArgs{}, y0q);
    if (e != cudaSuccess) return e;
    // pass 2: S_in(k + 1) = S_in(k) M_k + E_k for k = 1 .. nseg - 1, from S_in(1) = E_0
    e = launch_combine(B, H, nseg - 1, em, false, em + zst, zst, em + (nseg + 1) * zst, zst, sin, zst, st);
    if (e != cudaSuccess) return e;
    // pass 3: y of segments 1 .. nseg - 1, and the final state
    e = launch_fixup(B, T, H, t_seg, 1, nseg, y_dt, y0q, sin, zst, y, st);
    if (e != cudaSuccess || sT == nullptr) return e;
    return cudaMemcpyAsync(sT, sin + (nseg - 1) * zst, zst * sizeof(float), cudaMemcpyDeviceToDevice, st);
}

cudaError_t fwd_chunk(int B, int T, int H, wkv7_dtype y_dt, const void *r, const void *w, const void *k,
                      const void *v, const void *a, const void *b, const float *s0, void *y, float *sT,
                      int nseg, void *workspace, long long wait_limit, cudaStream_t st, float *ckpt,
                      const EpiArgs &epi, bool fixup, uint4 *mq) {
    if (fixup && nseg > 1 && ckpt == nullptr && epi.rho == nullptr && y != nullptr)
        return fwd_chunk_fixup(B, T, H, y_dt, r, w, k, v, a, b, s0, y, sT, nseg, workspace, wait_limit, st);
    if (nseg <= 1)
        return launch_chunk(B, T, H, T, 1, 1, y_dt, r, w, k, v, a, b, s0, 0, y, sT, 0, -1, wait_limit, st, ckpt, 0,
                            epi, mq);
    int t_seg;
    seg_split(T, nseg, t_seg, nseg);
    if (nseg <= 1)
        return launch_chunk(B, T, H, T, 1, 1, y_dt, r, w, k, v, a, b, s0, 0, y, sT, 0, -1, wait_limit, st, ckpt, 0,
                            epi, mq);
    const long long zst = (long long)B * H * kN * kN;
    float *em = static_cast<float *>(workspace);                // [2 (nseg-1)][B][H][64][64]
    float *sin = em + (size_t)2 * (nseg - 1) * zst;             // [nseg - 1][B][H][64][64]
    // pass 1: one dual launch over segments 0..nseg-2.  Segment 0 starts
    // from s0 and writes its y (and checkpoints): its E is the entry state of
    // segment 1.  Segments k >= 1 give E_k (from 0) and M_k (from I, v = 0).
    cudaError_t e = launch_dual(B, T, H, t_seg, nseg - 1, r, w, k, v, a, b, em, zst, em + (size_t)(nseg - 1) * zst,
                                zst, wait_limit, st, y, y_dt, s0, ckpt, epi, nullptr, mq);
    if (e != cudaSuccess) return e;
    // pass 2: entry states of segments 1..nseg-1, from segment 1's
    e = launch_combine(B, H, nseg - 2, em, false, em + zst, zst, em + (size_t)nseg * zst, zst, sin, zst, st);
    if (e != cudaSuccess) return e;
    // pass 3: segments 1..nseg-1 from their true entry states; the last one writes sT
    return launch_chunk(B, T, H, t_seg, nseg - 1, nseg - 1, y_dt, r, w, k, v, a, b, sin, zst, y, sT, 0, nseg - 2,
                        wait_limit, st, ckpt, 1, epi, mq);
}

}  // namespace wkv7
