// Chunk gradients of the WKV7 backward on the sm_100a tensor cores (tcgen05).
//
// Same algebra as bwd_chunk_kernel (the adjoint of the chunked form, see
// bwd_chunk.cu), for bf16 inputs: per chunk of L = 32 tokens, given the entry
// state S_in and dS = dL/dS at the chunk end, with the suffix decay products
// p_t = prod_{m >= t} w_m (p_32 = 1, G = p_0):
//   a' = a / p_t,  r' = r / p_{t+1},  b- = b p_{t+1},  k- = k p_{t+1},  SG = S_in diag(G)
//   L_xy[t][s] = x'_t . y-_s  (ab, ak: s < t;  rb, rk: s <= t),  T = (I - L_ab)^{-1}
//   Z = a' SG^T + L_ak V,  U = T Z,  dU = b- dS^T + L_rb^T dY,  dZ = T^T dU
//   dV = k- dS^T + L_rk^T dY + L_ak^T dZ,  dL = [dY; dZ] [U; V]^T (masked)
//   [dr'; da'] = [dY; dZ] SG + dL [b-; k-],   [db'; dk'] = [U; V] dS + dL^T [r'; a']
//   da = da' / p_t,  dr = dr' / p_{t+1},  db = db' p_{s+1},  dk = dk' p_{s+1}
//   q_t = dr r - db b - dk k + (da a)_{t+1} + [t = L-1] sum_i S_out dS,  dw_m = sum_{t>=m} q_t / w_m
//
// Every product is an M=128 tensor-core product with one output row per TMEM
// lane; unrelated products share one instruction by stacking their operands
// along M and N (the off-diagonal blocks of such a product are computed and
// ignored: an MMA costs the same whatever it holds).  Five rounds:
//   A  Gram: X X^T with X = [r'; a'; b-; k-] (128 x 64): L_rb, L_rk, L_ab, L_ak
//      and their transposes in one product
//   B  [SG; dS] [a'; b-; k-]^T + [V^T; dY^T] [L_ak; L_rb^T]^T
//      -> Z^T (lanes 0-63, cols 0-31), dU^T (lanes 64-127, cols 32-63),
//         the k- dS^T part of dV^T (lanes 64-127, cols 64-95)
//   C  [T; T^T] [Z^T; dU^T]^T -> U (lanes 0-31), dZ (lanes 32-63)
//   D  ZYUV ZYUV^T with ZYUV = [dY; dZ; U; V] -> dL (lanes 0-63, cols 64-127)
//      and dL^T (lanes 64-127, cols 0-63);  dV^T += [dY; dZ]^T [L_rk; L_ak]
//   E  ZYUV [SG | dS] + [dL; dL^T] [[b-; k-] | [r'; a']] -> [dr'; da'] (lanes
//      0-63, cols 0-63) and [db'; dk'] (lanes 64-127, cols 64-127); the B
//      operands are side-by-side copies ([SG | dS] made in P3 by the warps
//      that idle there, so the first half is issued after round D and runs
//      under P4)
// Operands are bf16 hi/lo splits (three passes, two when one side is an exact
// bf16 input: v, dy), accumulation in fp32 in TMEM.  The CUDA cores prepare
// the operands, invert the 32 x 32 unit lower triangular I - L_ab by 16 x 16
// blocks, move results between rounds and finish the gradients.
//
// A persistent grid, one CTA per SM walking the chunks: warps 0-15 compute
// (four per TMEM lane quadrant, each taking 16 of an accumulator's columns:
// the chunk's phases are short dependent sequences, and two warps per
// scheduler left most issue slots idle), warp 16 issues the tensor-core
// rounds; hand-offs through named barriers
// (ready: compute -> issuer, done: issuer -> compute), every wait of the issuer
// bounded.  The next chunk's token tiles arrive by cp.async into the raw tile
// buffer (read only in the first phase), issued while the compute warps wait
// for round C; its S_in and dS into the [SG; dS] tiles' space (last read in
// P3), issued while they wait for round D; its states are pulled into L2 one
// chunk ahead.
#include "umma.cuh"

namespace wkv7 {

namespace bwtc {

constexpr int L = 32;
constexpr int NCW = 16;                  // compute warps: four per TMEM lane quadrant
constexpr int NC = 32 * NCW, NT = NC + 32;
constexpr uint32_t TMEM_COLS = 512;
// TMEM columns
constexpr uint32_t CA = 0;       // round A (128), later round D's dL block (128)
constexpr uint32_t CB = 128;     // round B (96): Z^T | dU^T | dV^T
constexpr uint32_t CC = 256;     // round C (128), later the dL stack as A operand (hi 256, lo 288)
constexpr uint32_t CE = 384;     // round E (128)
constexpr uint32_t ADL_HI = 256, ADL_LO = 288;

// shared memory (bytes); bf16 tiles in core-matrix layout, hi and lo copies
constexpr uint32_t X1_HI = 0, X1_LO = 16384;          // [128][64]: r', a', b-, k- rows
constexpr uint32_t SGD_HI = 32768, SGD_LO = 49152;    // [128][64]: SG rows i, dS rows i
constexpr uint32_t ZY_HI = 65536, ZY_LO = 81920;      // [128][64]: dY, dZ, U, V rows
constexpr uint32_t VYZ_HI = 98304, VYZ_LO = 114688;   // [64][128]: rows t: [V | dY], then [0 | dZ]
constexpr uint32_t ZDU_HI = 131072, ZDU_LO = 139264;  // [128][32]: Z^T rows i, dU^T rows i
constexpr uint32_t LB2_HI = 147456, LB2_LO = 151552;  // [64][32]: L_ak rows t, L_rb^T rows s
constexpr uint32_t TT_HI = 155648, TT_LO = 159744;    // [64][32]: T rows t, T^T rows s
constexpr uint32_t LRK_HI = 163840, LRK_LO = 167936;  // [64][32]: L_rk rows t, L_ak rows t
// token rows of the raw inputs and of p_t are padded (144 B, 68 floats) so
// that a warp reading one row per lane spreads over the banks
constexpr int RAWP = 72;                              // bf16 per raw row
constexpr uint32_t RAW = 172032;                      // bf16 [7][32][72]: r w k v a b dy
constexpr int LDP = 68;
constexpr uint32_t PSM = RAW + 7 * 32 * RAWP * 2;     // fp32 [33][68]: p_t
constexpr int LDT = 36;
constexpr uint32_t LABT = PSM + 33 * LDP * 4;         // fp32 [32][36]: L_ab^T (row s, col t)
constexpr int LDTS = 33;
constexpr uint32_t TSM = LABT + 32 * LDT * 4;         // fp32 [32][33]: T
constexpr uint32_t ZSM = TSM + 32 * LDTS * 4;         // fp32 [16][16]
// round E's side-by-side B operands: [SG | dS] after round C (ZDU, LB2, TT are
// no longer read), so that round E's first half can run under P4;
// [[b-; k-] | [r'; a']] after round D (VYZ is no longer read)
constexpr uint32_t SGDC_HI = ZDU_HI, SGDC_LO = ZDU_HI + 16384;   // [64][128]: rows i: [SG | dS]
constexpr uint32_t X1C_HI = VYZ_HI, X1C_LO = VYZ_LO;             // [64][128]: rows: [[b-; k-] | [r'; a']]
// after round E: fp32 scratch of the q and dw sums
constexpr int LDQ = 68;
constexpr uint32_t CQ = VYZ_HI;                       // fp32 [4][32][68]: q terms of dr, da, db, dk
constexpr uint32_t DWTOT = CQ + 4 * 32 * LDQ * 4;     // fp32 [8][64]: token-block sums of q
constexpr uint32_t GSTG = DWTOT + 8 * 64 * 4;         // the four gradient tiles, rows padded by 16 B (<= 34816 B)
static_assert(GSTG + 4 * 32 * (64 * 4 + 16) <= RAW, "gradient staging ends before the token tiles");
constexpr uint32_t BAR = ZSM + 1024;                  // 6 mbarriers: rounds A..E, round E's first half
constexpr uint32_t TMEM_SLOT = BAR + 48;
constexpr uint32_t FLAG = BAR + 52;
constexpr uint32_t CPART = BAR + 64;                  // fp32 [8][64]: sums of S_out dS per 8 rows (P0b -> P5)
constexpr uint32_t SMEM_BYTES = CPART + 8 * 64 * 4;
// staged states (fp32, row-major) arriving by cp.async: the chunk's S_in and
// dS into the [SG; dS] tiles' space, issued under the previous chunk's round
// D (P3 was its last reader); S_out, rows 0-31 and 32-63, at the top of the
// chunk into the halves of VYZ that nothing reads before P3
constexpr uint32_t ST_SIN = SGD_HI, ST_DS = SGD_LO;
constexpr uint32_t ST_SOUT0 = VYZ_HI + 8192, ST_SOUT1 = VYZ_LO + 8192;
// A staged state row (64 floats, 16 chunks of 16 bytes) keeps chunk g at
// position g ^ (row % 8): the readers take four chunks of 8 rows per warp,
// which then fall on distinct banks (unswizzled, the 256-byte rows put all 8
// rows on the same banks).
__device__ __forceinline__ uint32_t st_off(int row, int g) { return (uint32_t)(row * 256 + ((g ^ (row & 7)) << 4)); }

constexpr uint32_t BAR_READY = 2, BAR_DONE = 7;      // named barriers 2-6, 7-11
constexpr long long kDrainCycles = 200000000LL;
constexpr float kMinDecay = 1e-30f;

enum { TR = 0, TW = 1, TK = 2, TV = 3, TA = 4, TB = 5, TDY = 6 };

__device__ __forceinline__ void csync() { umma::named_sync(1, NC); }

}  // namespace bwtc

__device__ __forceinline__ void bwtc_prefetch_l2(const void *p, uint32_t bytes) {
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

// 16 fp32 values -> 8 bf16 pairs (hi) and 8 (lo), packed per 32-bit word (even index in the low half)
__device__ __forceinline__ void bwtc_pack16(const float *x, uint32_t *ph, uint32_t *pl) {
#pragma unroll
    for (int e2 = 0; e2 < 8; ++e2) {
        const float x0 = x[2 * e2], x1 = x[2 * e2 + 1];
        const __nv_bfloat162 hp = __floats2bfloat162_rn(x0, x1);
        const uint32_t hu = *reinterpret_cast<const uint32_t *>(&hp);
        const __nv_bfloat162 lp = __floats2bfloat162_rn(x0 - __uint_as_float(hu << 16),
                                                        x1 - __uint_as_float(hu & 0xffff0000u));
        ph[e2] = hu;
        pl[e2] = *reinterpret_cast<const uint32_t *>(&lp);
    }
}

template <typename GradT>
__global__ void __launch_bounds__(bwtc::NT, 1)
bwd_chunk_tc_kernel(int T, int H, const __nv_bfloat16 *__restrict__ r, const __nv_bfloat16 *__restrict__ w,
                    const __nv_bfloat16 *__restrict__ k, const __nv_bfloat16 *__restrict__ v,
                    const __nv_bfloat16 *__restrict__ a, const __nv_bfloat16 *__restrict__ b,
                    const __nv_bfloat16 *__restrict__ dy, const float *__restrict__ ckpt,
                    const float *__restrict__ sfin, const float *__restrict__ dS_out, GradT *__restrict__ dr,
                    GradT *__restrict__ dw, GradT *__restrict__ dk, GradT *__restrict__ dv,
                    GradT *__restrict__ da, GradT *__restrict__ db, long long wait_limit, int total) {
    using namespace bwtc;
    using namespace umma;
    extern __shared__ __align__(1024) unsigned char sm[];
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int nck = (T + L - 1) / L;
    const size_t tok_stride = (size_t)H * kN;
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(sm + FLAG);
    auto done_bar = [&](int rd) { return sbase + BAR + 8u * (uint32_t)rd; };
    int last_rd = -1;
    uint32_t last_par = 0;
    // chunk id -> (head, chunk): tokens in it, offset of its first token, its states
    auto chunk_len = [&](int id) { return min(L, T - (id % nck) * L); };
    auto chunk_base = [&](int id) {
        const int head = id / nck;
        return (((size_t)(head / H) * T + (size_t)(id % nck) * L) * H + head % H) * kN;
    };

    // The token tiles of a chunk (r w k v a b dy) go to RAW by cp.async one
    // chunk ahead, once the current chunk's tiles have been read (RAW is read
    // only at the start of a chunk); thread -> (token tid / 8,
    // channels 8 (tid % 8) ..).  Rows past the end are no-op tokens (w = 1,
    // the rest 0), written directly.
    auto issue_tiles = [&](int id) {
        if (id < total && tid < 256) {
            const int t = tid >> 3, ch = tid & 7;
            unsigned char *dst = sm + RAW + (t * RAWP + 8 * ch) * 2;
            constexpr uint32_t TEN = L * RAWP * 2;           // bytes per tensor tile
            if (t < chunk_len(id)) {
                const size_t bs = chunk_base(id) + (size_t)t * tok_stride + 8 * ch;
                cp_async16(dst + TR * TEN, r + bs);
                cp_async16(dst + TW * TEN, w + bs);
                cp_async16(dst + TK * TEN, k + bs);
                cp_async16(dst + TV * TEN, v + bs);
                cp_async16(dst + TA * TEN, a + bs);
                cp_async16(dst + TB * TEN, b + bs);
                cp_async16(dst + TDY * TEN, dy + bs);
            } else {
                const uint4 zero = make_uint4(0, 0, 0, 0);
#pragma unroll
                for (int ten = 0; ten < 7; ++ten)
                    *reinterpret_cast<uint4 *>(dst + ten * TEN) =
                        ten == TW ? make_uint4(0x3f803f80u, 0x3f803f80u, 0x3f803f80u, 0x3f803f80u) : zero;
            }
        }
        cp_async_commit();
    };
    // The states a chunk reads (S_in, dS, S_out: 16 KB each) are pulled into
    // L2 one chunk ahead, then staged in shared memory by cp.async.
    auto s_out_of = [&](int id) {
        return (id % nck) + 1 < nck ? ckpt + (size_t)(id + 1) * kN * kN : sfin + (size_t)(id / nck) * kN * kN;
    };
    // S_out of a chunk into ST_SOUT0 / ST_SOUT1 (compute threads, 2 x 16 B each)
    auto issue_sout = [&](int id) {
        const float *src = s_out_of(id);
        for (int x = tid; x < 1024; x += NC)   // chunk x: row x / 16, chunk x % 16
            cp_async16(sm + (x < 512 ? ST_SOUT0 : ST_SOUT1) + st_off((x >> 4) & 31, x & 15), src + 4 * x);
        cp_async_commit();
    };
    // S_in and dS of a chunk into ST_SIN / ST_DS (compute threads, 4 x 16 B each)
    auto issue_states = [&](int id) {
        if (id < total) {
            for (int x = tid; x < 2048; x += NC) {
                const int which = x >> 10, o4 = 4 * (x & 1023);
                const float *src = (which ? dS_out : ckpt) + (size_t)id * kN * kN + o4;
                cp_async16(sm + (which ? ST_DS : ST_SIN) + st_off(o4 >> 6, (o4 & 63) >> 2), src);
            }
        }
        cp_async_commit();
    };
    auto prefetch_states = [&](int id) {
        if (id >= total || tid >= 3) return;
        const float *p = tid == 0 ? ckpt + (size_t)id * kN * kN : tid == 1 ? dS_out + (size_t)id * kN * kN : s_out_of(id);
        bwtc_prefetch_l2(p, kN * kN * sizeof(float));
    };

    // ---- set-up (once per CTA) ------------------------------------------------------------
    if (tid == 0) {
        for (int rd = 0; rd < 6; ++rd) mbar_init(done_bar(rd), 1);
        *abort_flag = 0;
    }
    if (warp == NCW) tmem_alloc(sbase + TMEM_SLOT, TMEM_COLS);
    if (tid < NC) {
        issue_tiles(blockIdx.x);
        issue_states(blockIdx.x);
        prefetch_states(blockIdx.x);
        for (int x = tid; x < 256; x += NC) {          // ZYUV lo rows 0-31 (dY) and 96-127 (V): exact, 4 KB each
            *reinterpret_cast<uint4 *>(sm + ZY_LO + 16 * x) = make_uint4(0, 0, 0, 0);
            *reinterpret_cast<uint4 *>(sm + ZY_LO + 12288 + 16 * x) = make_uint4(0, 0, 0, 0);
        }
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + TMEM_SLOT);

    if (warp == NCW) {
        // ================= MMA issuer =================
        const uint32_t id_a = idesc_bf16(128, 128, 0, 0);
        const uint32_t id_b1 = idesc_bf16(128, 96, 0, 0);
        const uint32_t id_b2 = idesc_bf16(128, 64, 1, 0);
        const uint32_t id_c = idesc_bf16(128, 128, 0, 0);
        const uint32_t id_d2 = idesc_bf16(128, 32, 1, 1);
        const OpD x1 = opd_k(sbase + X1_HI, sbase + X1_LO, 64);                     // [r'; a'; b-; k-], K = j
        const OpD x1_abk = opd_k(sbase + X1_HI + 4096, sbase + X1_LO + 4096, 64);   // [a'; b-; k-]
        const OpD sgd = opd_k(sbase + SGD_HI, sbase + SGD_LO, 64);                  // [SG; dS], K = j
        const OpD vy = opd_mn(sbase + VYZ_HI, 0, 128);                              // [V^T; dY^T], K = t < 32, exact
        const OpD vyz = opd_mn(sbase + VYZ_HI, sbase + VYZ_LO, 128);                // lanes 64-127: [dY; dZ]^T, K = t'
        const OpD lb2 = opd_k(sbase + LB2_HI, sbase + LB2_LO, 32);                  // [L_ak; L_rb^T]
        const OpD tt = opd_k(sbase + TT_HI, sbase + TT_LO, 32);                     // [T; T^T]
        const OpD zdu = opd_k(sbase + ZDU_HI, sbase + ZDU_LO, 32);                  // [Z^T; dU^T]
        const OpD zy = opd_k(sbase + ZY_HI, sbase + ZY_LO, 64);                     // [dY; dZ; U; V], K = i
        const OpD lrk = opd_mn(sbase + LRK_HI, sbase + LRK_LO, 32);                 // [L_rk; L_ak], K = t'
        const uint32_t id_e = idesc_bf16(128, 128, 0, 1);
        const OpD sgdc = opd_mn(sbase + SGDC_HI, sbase + SGDC_LO, 128);             // [SG | dS], K = i
        const OpD x1c = opd_mn(sbase + X1C_HI, sbase + X1C_LO, 128);                // [[b-; k-] | [r'; a']], K = s', t'
        // one round: wait for the hand-over, issue, commit, wait for the
        // commit, release the compute warps, then issue any work that runs on
        // under the next compute phase (with its own commit, so that a drain
        // after an abort covers it); every barrier is passed once whatever
        // happens, nothing is issued after a wait gave up.  Issuing blocks
        // while the tensor pipe is busy, so the extra work goes in only after
        // the round's completion has been handed over.
        uint32_t par = 0;                            // phase parity of this chunk's round barriers
        auto nothing = [] { return false; };
        auto round = [&](int rd, auto &&issue, auto &&more) {
            named_sync(BAR_READY + rd, NT);
            fence_after_sync();
            if (lane == 0 && *abort_flag == 0u) {
                issue();
                commit(done_bar(rd));
                last_rd = rd;
                last_par = par;
                if (!mbar_spin_abortable(done_bar(rd), par, wait_limit, abort_flag)) *abort_flag = 1;
            }
            __syncwarp();
            fence_before_sync();
            named_arrive(BAR_DONE + rd, NT);
            if (lane == 0 && *abort_flag == 0u && more()) {
                commit(done_bar(5));
                last_rd = 5;
            }
            __syncwarp();
        };
        for (int id = blockIdx.x, it = 0; id < total; id += gridDim.x, ++it) {
            par = (uint32_t)it & 1u;
            round(0, [&] { gemm_split_d(tmem + CA, x1, x1, id_a, 4, false); }, nothing);
            round(1, [&] {
                gemm_split_d(tmem + CB, sgd, x1_abk, id_b1, 4, false);
                gemm_split_d(tmem + CB, vy, lb2, id_b2, 2, true);
            }, nothing);
            round(2, [&] { gemm_split_d(tmem + CC, tt, zdu, id_c, 2, false); }, nothing);
            round(3, [&] {
                gemm_split_d(tmem + CA, zy, zy, id_a, 4, false);
                gemm_split_d(tmem + CB + 64, vyz, lrk, id_d2, 4, true);
            }, [&] {                                 // round E's first half, ZYUV [SG | dS], under P4
                gemm_split_d(tmem + CE, zy, sgdc, id_e, 4, false);
                return true;
            });
            round(4, [&] { gemm_split_ts(tmem + CE, tmem + ADL_HI, tmem + ADL_LO, x1c, id_e, 4, true); }, nothing);
        }
        __syncwarp();
    } else {
        // ================= compute warps =================
        // TMEM lane quadrant, column half, and which half of that half (the
        // four warps of a quadrant split an accumulator's columns)
        const int q4 = warp & 3, hc = (warp >> 2) & 1, part = warp >> 3;
        const uint32_t quad = (uint32_t)(32 * q4) << 16;
        auto ready_arrive = [&](int rd) {
            fence_smem_to_async();
            fence_before_sync();
            named_arrive(BAR_READY + rd, NT);
        };
        auto done_wait = [&](int rd) {
            named_sync(BAR_DONE + rd, NT);
            fence_after_sync();
        };
        float *psm = reinterpret_cast<float *>(sm + PSM);
        for (int id = blockIdx.x; id < total; id += gridDim.x) {
            const int Lc = chunk_len(id);
            const size_t base = chunk_base(id);
            csync();                                 // the previous chunk's last reads are done
            issue_sout(id);
            // zero the lo copy of dY in VYZ (rows 0-31, columns 64-127; dY is
            // exact), which round D reads; columns 0-63 of VYZ feed only
            // accumulator lanes that are never read, and rows 32-63 take dZ
            if (tid < 256) {                             // lane -> row: a quarter-warp fills one core matrix
                const int t = tid & 31, ch = tid >> 5;
                *reinterpret_cast<uint4 *>(sm + VYZ_LO + cm_off(t, 64 + 8 * ch, 128)) = make_uint4(0, 0, 0, 0);
            }
            cp_async_wait<1>();                      // this chunk's token tiles, S_in and dS (not yet S_out)
            csync();
            // ---- P0a: suffix decay products and the decayed operands (warps 0-7:
            //      warp -> 8 channels, lane -> token; 16-byte accesses, so that a
            //      quarter-warp's 8 tokens fall on distinct banks) ----
            if (warp < 8) {
                const int g = warp, t = lane;
                auto ld8 = [&](int ten, float *o) {
                    const uint4 u = *reinterpret_cast<const uint4 *>(sm + RAW + ((ten * L + t) * RAWP + 8 * g) * 2);
                    const uint32_t uu[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                    for (int q = 0; q < 4; ++q) {
                        o[2 * q] = __uint_as_float(uu[q] << 16);
                        o[2 * q + 1] = __uint_as_float(uu[q] & 0xffff0000u);
                    }
                };
                float inc[8];                            // p_t = prod_{m >= t} w_m
                ld8(TW, inc);
#pragma unroll
                for (int o = 1; o < 32; o <<= 1)
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float up = __shfl_down_sync(0xffffffffu, inc[e], o);
                        if (lane + o < 32) inc[e] *= up;
                    }
                *reinterpret_cast<float4 *>(psm + t * LDP + 8 * g) = make_float4(inc[0], inc[1], inc[2], inc[3]);
                *reinterpret_cast<float4 *>(psm + t * LDP + 8 * g + 4) = make_float4(inc[4], inc[5], inc[6], inc[7]);
                if (lane == 31) {
                    *reinterpret_cast<float4 *>(psm + L * LDP + 8 * g) = make_float4(1.f, 1.f, 1.f, 1.f);
                    *reinterpret_cast<float4 *>(psm + L * LDP + 8 * g + 4) = make_float4(1.f, 1.f, 1.f, 1.f);
                }
                float nxt[8];                            // p_{t+1}
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float n1 = __shfl_down_sync(0xffffffffu, inc[e], 1);
                    nxt[e] = lane == 31 ? 1.f : n1;
                    if (lane == 0 && inc[e] < kMinDecay) raise_status(WKV7_ERR_RANGE);
                }
                // one operand at a time (loaded just before use: fewer live registers)
                {
                    float v[8], x[8];
                    ld8(TR, v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = __fdividef(v[e], nxt[e]);
                    store8_split(sm + X1_HI, sm + X1_LO, cm_off(t, 8 * g, 64), x);
                    ld8(TA, v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = __fdividef(v[e], inc[e]);
                    store8_split(sm + X1_HI, sm + X1_LO, cm_off(32 + t, 8 * g, 64), x);
                    ld8(TB, v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = v[e] * nxt[e];
                    store8_split(sm + X1_HI, sm + X1_LO, cm_off(64 + t, 8 * g, 64), x);
                    ld8(TK, v);
#pragma unroll
                    for (int e = 0; e < 8; ++e) x[e] = v[e] * nxt[e];
                    store8_split(sm + X1_HI, sm + X1_LO, cm_off(96 + t, 8 * g, 64), x);
                }
                // exact bf16 operands: V, dY into VYZ rows t ([V | dY]) and ZYUV rows t (dY), 96 + t (V)
                const uint4 vraw = *reinterpret_cast<const uint4 *>(sm + RAW + ((TV * L + t) * RAWP + 8 * g) * 2);
                const uint4 yraw = *reinterpret_cast<const uint4 *>(sm + RAW + ((TDY * L + t) * RAWP + 8 * g) * 2);
                *reinterpret_cast<uint4 *>(sm + VYZ_HI + cm_off(t, 8 * g, 128)) = vraw;
                *reinterpret_cast<uint4 *>(sm + VYZ_HI + cm_off(t, 64 + 8 * g, 128)) = yraw;
                *reinterpret_cast<uint4 *>(sm + ZY_HI + cm_off(t, 8 * g, 64)) = yraw;
                *reinterpret_cast<uint4 *>(sm + ZY_HI + cm_off(96 + t, 8 * g, 64)) = vraw;
            }
            ready_arrive(0);                                     // round A: X1
            csync();                                             // p_t visible; RAW no longer read
            // ---- P0b: SG = S_in diag(G) (rows 0-63) and dS (rows 64-127); thread ->
            //      row 8 (tid / 64) + tid % 8, columns 8 ((tid / 8) % 8) ..: a quarter-warp
            //      takes 8 rows of one column group, 16-byte accesses on distinct banks ----
            {
                const int rb = tid >> 6, i = 8 * rb + (tid & 7), c0 = 8 * ((tid >> 3) & 7);
                float sg[8], dsv[8];
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const uint32_t so4 = st_off(i, (c0 >> 2) + u);
                    const float4 s4 = *reinterpret_cast<const float4 *>(sm + ST_SIN + so4);
                    const float4 d4 = *reinterpret_cast<const float4 *>(sm + ST_DS + so4);
                    const float4 p4 = *reinterpret_cast<const float4 *>(psm + c0 + 4 * u);   // G = p_0
                    sg[4 * u] = s4.x * p4.x; sg[4 * u + 1] = s4.y * p4.y;
                    sg[4 * u + 2] = s4.z * p4.z; sg[4 * u + 3] = s4.w * p4.w;
                    dsv[4 * u] = d4.x; dsv[4 * u + 1] = d4.y; dsv[4 * u + 2] = d4.z; dsv[4 * u + 3] = d4.w;
                }
                cp_async_wait<0>();                      // S_out
                csync();                                 // the staged states are read before SGD replaces them
                store8_split(sm + SGD_HI, sm + SGD_LO, cm_off(i, c0, 64), sg);
                store8_split(sm + SGD_HI, sm + SGD_LO, cm_off(64 + i, c0, 64), dsv);
                // the chunk's last token also scales S_out: q_{Lc-1} += sum_i S_out dS
                // (the 8 rows of a quarter-warp summed by shuffles, then partial sums
                // per block of 8 rows)
                float cs[8];
                const uint32_t so = i < 32 ? ST_SOUT0 : ST_SOUT1;
#pragma unroll
                for (int u = 0; u < 2; ++u) {
                    const float4 s4 = *reinterpret_cast<const float4 *>(sm + so + st_off(i & 31, (c0 >> 2) + u));
                    cs[4 * u] = s4.x * dsv[4 * u]; cs[4 * u + 1] = s4.y * dsv[4 * u + 1];
                    cs[4 * u + 2] = s4.z * dsv[4 * u + 2]; cs[4 * u + 3] = s4.w * dsv[4 * u + 3];
                }
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 1);
                    cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 2);
                    cs[e] += __shfl_xor_sync(0xffffffffu, cs[e], 4);
                }
                if ((lane & 7) == 0) {
                    float *cp = reinterpret_cast<float *>(sm + CPART) + rb * kN + c0;
                    *reinterpret_cast<float4 *>(cp) = make_float4(cs[0], cs[1], cs[2], cs[3]);
                    *reinterpret_cast<float4 *>(cp + 4) = make_float4(cs[4], cs[5], cs[6], cs[7]);
                }
            }

            // ---- P1: Gram rows -> L tiles (lane = row of X X^T; the two warps of a
            //      role take 16 of its 32 columns each) ----
            done_wait(0);
            {
                const int lr = lane, e0 = 16 * part;     // token t (quadrants 0, 1) or s (quadrant 2)
                if (q4 == 0 && hc == 1) {                // r'_t . k-_s: L_rk rows t (s <= t)
                    float x[16];
                    tmem_ld16(tmem + quad + CA + 96 + e0, x);
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] = e0 + e <= lr ? x[e] : 0.f;
#pragma unroll
                    for (int u = 0; u < 2; ++u)
                        store8_split(sm + LRK_HI, sm + LRK_LO, cm_off(lr, e0 + 8 * u, 32), x + 8 * u);
                } else if (q4 == 1 && hc == 1) {         // a'_t . k-_s: L_ak rows t (s < t)
                    float x[16];
                    tmem_ld16(tmem + quad + CA + 96 + e0, x);
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] = e0 + e < lr ? x[e] : 0.f;
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        store8_split(sm + LB2_HI, sm + LB2_LO, cm_off(lr, e0 + 8 * u, 32), x + 8 * u);
                        store8_split(sm + LRK_HI, sm + LRK_LO, cm_off(32 + lr, e0 + 8 * u, 32), x + 8 * u);
                    }
                } else if (q4 == 2 && hc == 0) {         // b-_s . r'_t: L_rb^T rows s (t >= s)
                    float x[16];
                    tmem_ld16(tmem + quad + CA + 0 + e0, x);
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] = e0 + e >= lr ? x[e] : 0.f;
#pragma unroll
                    for (int u = 0; u < 2; ++u)
                        store8_split(sm + LB2_HI, sm + LB2_LO, cm_off(32 + lr, e0 + 8 * u, 32), x + 8 * u);
                } else if (q4 == 2 && hc == 1) {         // b-_s . a'_t: L_ab^T rows s (t > s), fp32
                    float x[16];
                    tmem_ld16(tmem + quad + CA + 32 + e0, x);
                    float *dst = reinterpret_cast<float *>(sm + LABT) + lr * LDT + e0;
#pragma unroll
                    for (int e4 = 0; e4 < 4; ++e4) {
                        const int t0 = e0 + 4 * e4;
                        *reinterpret_cast<float4 *>(dst + 4 * e4) =
                            make_float4(t0 + 0 > lr ? x[4 * e4 + 0] : 0.f, t0 + 1 > lr ? x[4 * e4 + 1] : 0.f,
                                        t0 + 2 > lr ? x[4 * e4 + 2] : 0.f, t0 + 3 > lr ? x[4 * e4 + 3] : 0.f);
                    }
                }
            }
            ready_arrive(1);                             // round B: SG, dS, a', b-, k-, V, dY, L_ak, L_rb^T
            csync();                                     // L_ab^T visible
            // ---- P1b: T = (I - L_ab)^{-1} by 16 x 16 blocks (fp32), then [T; T^T] ----
            {
                const float *labt = reinterpret_cast<const float *>(sm + LABT);
                float *ts = reinterpret_cast<float *>(sm + TSM);
                float *zs = reinterpret_cast<float *>(sm + ZSM);
                if (warp == 0) {                         // diagonal blocks, one column s per lane
                    const int blk = lane >> 4, sub = lane & 15, s = 16 * blk + sub;
                    float acc[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) acc[e] = e == sub ? 1.f : 0.f;
#pragma unroll
                    for (int m = 0; m < 15; ++m) {
                        const float xm = acc[m];
                        const float *row = labt + (16 * blk + m) * LDT + 16 * blk;   // L_ab[16 blk + e][16 blk + m]
#pragma unroll
                        for (int e = m + 1; e < 16; ++e) acc[e] = fmaf(row[e], xm, acc[e]);
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e) ts[(16 * blk + e) * LDTS + s] = acc[e];
                } else if (warp == 1) {                  // upper-right block is zero
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const int x = lane + 32 * e;
                        ts[(x >> 4) * LDTS + 16 + (x & 15)] = 0.f;
                    }
                }
                csync();
                if (tid < 256) {                         // Z = L21 T11
                    const int t = tid >> 4, s = tid & 15;
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m) acc = fmaf(labt[m * LDT + 16 + t], ts[m * LDTS + s], acc);
                    zs[t * 16 + s] = acc;
                }
                csync();
                if (tid < 256) {                         // T21 = T22 Z
                    const int t = tid >> 4, s = tid & 15;
                    float acc = 0.f;
#pragma unroll
                    for (int m = 0; m < 16; ++m) acc = fmaf(ts[(16 + t) * LDTS + 16 + m], zs[m * 16 + s], acc);
                    ts[(16 + t) * LDTS + s] = acc;
                }
                csync();
                if (tid < 256) {                         // T rows t and T^T rows 32 + s of TT
                    // thread -> row (lane) and 8 columns (warp % 4) of T (warps 0-3)
                    // or of T^T (warps 4-7): a quarter-warp stores 8 rows of one
                    // core-matrix column, the fp32 reads spread over the banks
                    const int r = tid & 31, u = (tid >> 5) & 3;
                    float x[8];
                    if (tid < 128) {
#pragma unroll
                        for (int k = 0; k < 8; ++k) x[k] = ts[r * LDTS + 8 * u + k];
                        store8_split(sm + TT_HI, sm + TT_LO, cm_off(r, 8 * u, 32), x);
                    } else {
#pragma unroll
                        for (int k = 0; k < 8; ++k) x[k] = ts[(8 * u + k) * LDTS + r];
                        store8_split(sm + TT_HI, sm + TT_LO, cm_off(32 + r, 8 * u, 32), x);
                    }
                }
            }
            // ---- P2: Z^T (lanes 0-63) and dU^T (lanes 64-127) -> ZDU rows ----
            done_wait(1);
            if (part == 0) {                             // 8 warps: 16 columns each
                const int row = 32 * q4 + lane;
                const uint32_t col = CB + (q4 < 2 ? 0u : 32u) + 16u * (uint32_t)hc;
                uint32_t r0[16];
                tmem_ld16_nowait(tmem + quad + col, r0);
                tmem_wait();
                float x[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) x[e] = __uint_as_float(r0[e]);
                store8_split(sm + ZDU_HI, sm + ZDU_LO, cm_off(row, 16 * hc, 32), x);
                store8_split(sm + ZDU_HI, sm + ZDU_LO, cm_off(row, 16 * hc + 8, 32), x + 8);
            }
            ready_arrive(2);                             // round C: [T; T^T], [Z^T; dU^T]
            issue_tiles(id + gridDim.x);                 // the next chunk's token tiles, while round C runs
            prefetch_states(id + gridDim.x);             // the next chunk's states into L2, under round C
            // ---- P3: U rows (lanes 0-31), dZ rows (lanes 32-63) -> ZYUV, VYZ ----
            done_wait(2);
            if (q4 < 2) {
                const int t = lane, cb = 32 * hc + 16 * part;
                float x[16];
                tmem_ld16(tmem + quad + CC + (q4 == 0 ? 0u : 64u) + (uint32_t)cb, x);
                if (q4 == 0) {
#pragma unroll
                    for (int u = 0; u < 2; ++u)
                        store8_split(sm + ZY_HI, sm + ZY_LO, cm_off(64 + t, cb + 8 * u, 64), x + 8 * u);
                } else {
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        store8_split(sm + ZY_HI, sm + ZY_LO, cm_off(32 + t, cb + 8 * u, 64), x + 8 * u);
                        store8_split(sm + VYZ_HI, sm + VYZ_LO, cm_off(32 + t, 64 + cb + 8 * u, 128), x + 8 * u);
                    }
                }
            } else {                                     // the other eight warps: [SG | dS] side by side
                const int u = ((2 * hc + q4 - 2) + 4 * part) * 32 + lane;   // 0 .. 255; SG rows to columns 0-63, dS to 64-127
                for (int x = u; x < 2048; x += 256) {
                    const int blk = x >> 6, hl = (blk >> 4) & 1, G = blk & 15;
                    const uint32_t src = (hl ? SGD_LO : SGD_HI) + G * 1024;
                    const uint32_t dst = (hl ? SGDC_LO : SGDC_HI) + ((G & 7) * 16 + (G < 8 ? 0 : 8)) * 128;
                    *reinterpret_cast<uint4 *>(sm + dst + 16 * (x & 63)) =
                        *reinterpret_cast<const uint4 *>(sm + src + 16 * (x & 63));
                }
            }
            ready_arrive(3);                             // round D: ZYUV, VYZ, [L_rk; L_ak]
            csync();                                     // every warp's P3 reads of SGD are done
            issue_states(id + gridDim.x);                // S_in, dS of the next chunk, under round D

            // ---- P4: dV out; the masked dL block as round E's A operand in TMEM ----
            done_wait(3);
            {
                // first the TMEM traffic (round E's first half is starting up on the
                // tensor pipe; these loads and stores then wait less for it), then
                // dV out and the side-by-side copy.
                // lanes 0-63: dL rows t' (columns s' = 32 hc + 16 part + e at CA + 64 + s');
                // lanes 64-127: dL^T rows s' (columns t' = 32 hc + 16 part + e at CA + t').
                // Mask: t' < 32 (r' rows) keeps s <= t, t' >= 32 (a' rows) keeps s < t.
                const int e0 = 32 * hc + 16 * part;
                float x[16];
                tmem_ld16(tmem + quad + CA + (q4 < 2 ? 64u : 0u) + (uint32_t)e0, x);
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    int tp, t_, s_;
                    if (q4 < 2) { tp = 32 * q4 + lane; t_ = lane; s_ = (e0 + e) & 31; }
                    else { tp = e0 + e; t_ = (e0 + e) & 31; s_ = lane; }
                    const bool keep = tp < 32 ? s_ <= t_ : s_ < t_;
                    x[e] = keep ? x[e] : 0.f;
                }
                uint32_t ph[8], pl[8];
                bwtc_pack16(x, ph, pl);
                tmem_st8(tmem + quad + ADL_HI + (uint32_t)(e0 >> 1), ph);
                tmem_st8(tmem + quad + ADL_LO + (uint32_t)(e0 >> 1), pl);
                tmem_st_wait();
            }
            if (q4 >= 2 && part == 0) {                  // dV^T rows i, columns s = 16 hc ..
                const int i = 32 * (q4 - 2) + lane;
                uint32_t r0[16];
                tmem_ld16_nowait(tmem + quad + CB + 64 + 16 * hc, r0);
                tmem_wait();
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const int s_ = 16 * hc + e;
                    if (s_ < Lc) dv[base + (size_t)s_ * tok_stride + i] = from_f32<GradT>(__uint_as_float(r0[e]));
                }
            }
            // side-by-side copy for round E's second half: [[b-; k-] | [r'; a']]
            // from the X1 rows.  A group of 8 rows is 1 KB in both layouts (8
            // column chunks of 8 rows), so each moves as one contiguous block;
            // consecutive lanes move consecutive 16 bytes.
            for (int x = tid; x < 2048; x += NC) {
                const int blk = x >> 6, hl = (blk >> 4) & 1, G = blk & 15;
                const uint32_t src = (hl ? X1_LO : X1_HI) + G * 1024;
                const uint32_t dst = (hl ? X1C_LO : X1C_HI) + ((G & 7) * 16 + (G < 8 ? 8 : 0)) * 128;
                *reinterpret_cast<uint4 *>(sm + dst + 16 * (x & 63)) =
                    *reinterpret_cast<const uint4 *>(sm + src + 16 * (x & 63));
            }
            ready_arrive(4);                             // round E
            // ---- P5: the four gradients, q, dw ----
            done_wait(4);
            {
                const int rrow = lane;                   // token t (q4 0, 1) or s (q4 2, 3)
                const int j0 = 32 * hc + 16 * part;      // this warp's 16 channels
                float x[16];
                tmem_ld16(tmem + quad + CE + (q4 < 2 ? 0u : 64u) + (uint32_t)j0, x);
                // q terms, from the unscaled gradients and the decayed operands:
                // dr r = dr' r', da a = da' a', db b = db' b-, dk k = dk' k-
                // (X1 row 32 q4 + lane holds r', a', b-, k- for q4 = 0 .. 3);
                // + dr r, + da a (counted at t - 1), - db b, - dk k; zero on rows
                // past the end, whose decayed operands are zero
                {
                    float *cq = reinterpret_cast<float *>(sm + CQ) + (q4 * L + rrow) * LDQ + j0;
                    const float sign = q4 >= 2 ? -1.f : 1.f;
#pragma unroll
                    for (int u = 0; u < 2; ++u) {
                        const uint32_t off = cm_off(32 * q4 + rrow, j0 + 8 * u, 64);
                        const uint4 h8 = *reinterpret_cast<const uint4 *>(sm + X1_HI + off);
                        const uint4 l8 = *reinterpret_cast<const uint4 *>(sm + X1_LO + off);
                        const uint32_t hh[4] = {h8.x, h8.y, h8.z, h8.w}, ll[4] = {l8.x, l8.y, l8.z, l8.w};
                        float o8[8];
#pragma unroll
                        for (int q = 0; q < 4; ++q) {
                            o8[2 * q] = sign * x[8 * u + 2 * q] *
                                        (__uint_as_float(hh[q] << 16) + __uint_as_float(ll[q] << 16));
                            o8[2 * q + 1] = sign * x[8 * u + 2 * q + 1] *
                                            (__uint_as_float(hh[q] & 0xffff0000u) + __uint_as_float(ll[q] & 0xffff0000u));
                        }
                        *reinterpret_cast<float4 *>(cq + 8 * u) = make_float4(o8[0], o8[1], o8[2], o8[3]);
                        *reinterpret_cast<float4 *>(cq + 8 * u + 4) = make_float4(o8[4], o8[5], o8[6], o8[7]);
                    }
                }
                const float *prow = psm + (q4 == 1 ? rrow : rrow + 1) * LDP + j0;   // p_t for da, p_{t+1} else
                float pv[16];
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const float4 p4 = *reinterpret_cast<const float4 *>(prow + 4 * u);
                    pv[4 * u] = p4.x; pv[4 * u + 1] = p4.y; pv[4 * u + 2] = p4.z; pv[4 * u + 3] = p4.w;
                }
                if (q4 < 2) {                            // dr = dr' / p_{t+1},  da = da' / p_t
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] = __fdividef(x[e], pv[e]);
                } else {                                 // db, dk = (db', dk') p_{s+1}
#pragma unroll
                    for (int e = 0; e < 16; ++e) x[e] = x[e] * pv[e];
                }
                {   // into the staging tile of this gradient (row rrow, columns j0 ..); written out coalesced below
                    constexpr int PITCH = kN * (int)sizeof(GradT) + 16;
                    GradT *o = reinterpret_cast<GradT *>(sm + GSTG + (q4 * L + rrow) * PITCH) + j0;
#pragma unroll
                    for (int u = 0; u < 4; ++u)
                        store4(o + 4 * u, make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]));
                }
            }
            csync();
            {   // the four gradient tiles to global memory, 16 bytes per thread and step, a row per 8 or 16 threads
                constexpr int PITCH = kN * (int)sizeof(GradT) + 16;
                constexpr int CPR = kN * (int)sizeof(GradT) / 16;                // 16-byte chunks per row
                for (int x = tid; x < 4 * L * CPR; x += NC) {
                    const int ch = x % CPR, row = (x / CPR) % L, tile = x / (CPR * L);
                    GradT *g = tile == 0 ? dr : tile == 1 ? da : tile == 2 ? db : dk;
                    if (row < Lc)
                        *reinterpret_cast<uint4 *>(g + base + (size_t)row * tok_stride + ch * 16 / (int)sizeof(GradT)) =
                            *reinterpret_cast<const uint4 *>(sm + GSTG + (tile * L + row) * PITCH + 16 * ch);
                }
            }
            {   // dw_m = sum_{t >= m} q_t / w_m: thread -> column j, block of 4 tokens
                const float *cq = reinterpret_cast<const float *>(sm + CQ);
                const float *cp = reinterpret_cast<const float *>(sm + CPART);
                float *tot = reinterpret_cast<float *>(sm + DWTOT);
                const int j = tid & 63, blk = tid >> 6;
                float colsum = 0.f;
#pragma unroll
                for (int rb = 0; rb < 8; ++rb) colsum += cp[rb * kN + j];
                float loc[4], run = 0.f;
#pragma unroll
                for (int e = 3; e >= 0; --e) {
                    const int t = 4 * blk + e;
                    float q = cq[t * LDQ + j] + cq[(2 * L + t) * LDQ + j] + cq[(3 * L + t) * LDQ + j];
                    if (t + 1 < L) q += cq[(L + t + 1) * LDQ + j];
                    if (t == Lc - 1) q += colsum;
                    run += q;
                    loc[e] = run;
                }
                tot[blk * kN + j] = run;
                csync();
                float later = 0.f;
                for (int b2 = blk + 1; b2 < 8; ++b2) later += tot[b2 * kN + j];
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int t = 4 * blk + e;
                    if (t < Lc)
                        dw[base + (size_t)t * tok_stride + j] =
                            from_f32<GradT>(__fdividef((loc[e] + later) * psm[(t + 1) * LDP + j], psm[t * LDP + j]));
                }
            }
        }
    }

    // ---- tear-down ----------------------------------------------------------------------
    __syncthreads();
    if (*abort_flag) {
        // a wait gave up: report it, let the committed tensor-core work finish
        // (rounds complete in order), then release TMEM
        if (tid == 0) raise_status(WKV7_ERR_TIMEOUT);
        if (tid == NC && last_rd >= 0) mbar_wait(done_bar(last_rd), last_par, kDrainCycles);
        __syncthreads();
    }
    fence_after_sync();
    if (warp == NCW) tmem_dealloc(tmem, TMEM_COLS);
}

template <typename GradT>
cudaError_t launch_bwd_chunk_tc(int B, int T, int H, const void *r, const void *w, const void *k, const void *v,
                                const void *a, const void *b, const void *dy, const float *ckpt, const float *sfin,
                                const float *dS_out, void *dr, void *dw, void *dk, void *dv, void *da, void *db,
                                long long wait_limit, cudaStream_t st) {
    static_assert(bwtc::SMEM_BYTES <= 227 * 1024, "shared memory");
    const int nck = (T + bwtc::L - 1) / bwtc::L;
    const long long total = (long long)B * H * nck;   // chunks; one persistent CTA per SM walks them
    const int sms = current_sm_count();
    const int grid = (int)std::min<long long>(total, sms > 0 ? sms : 148);
    auto kern = bwd_chunk_tc_kernel<GradT>;
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bwtc::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    using bf = __nv_bfloat16;
    kern<<<grid, bwtc::NT, bwtc::SMEM_BYTES, st>>>(
        T, H, (const bf *)r, (const bf *)w, (const bf *)k, (const bf *)v, (const bf *)a, (const bf *)b,
        (const bf *)dy, ckpt, sfin, dS_out, (GradT *)dr, (GradT *)dw, (GradT *)dk, (GradT *)dv, (GradT *)da,
        (GradT *)db, wait_limit, (int)total);
    return cudaGetLastError();
}

// Chunk gradients on the tensor cores (bf16 inputs).
cudaError_t bwd_chunk_tc(int B, int T, int H, wkv7_dtype g_dt, const void *r, const void *w, const void *k,
                         const void *v, const void *a, const void *b, const void *dy, const float *ckpt,
                         const float *sfin, const float *dS_out, void *dr, void *dw, void *dk, void *dv, void *da,
                         void *db, long long wait_limit, cudaStream_t st) {
    if (g_dt == WKV7_F32)
        return launch_bwd_chunk_tc<float>(B, T, H, r, w, k, v, a, b, dy, ckpt, sfin, dS_out, dr, dw, dk, dv, da,
                                          db, wait_limit, st);
    return launch_bwd_chunk_tc<__nv_bfloat16>(B, T, H, r, w, k, v, a, b, dy, ckpt, sfin, dS_out, dr, dw, dk, dv,
                                              da, db, wait_limit, st);
}

}  // namespace wkv7
