// dL/dS at every chunk end from the chunks' transitions, on the tensor cores.
//
// Over a 32-token chunk c the recurrence (RWKV-7 "Goose" with Expressive
// Dynamic State Evolution: S_t = S_{t-1} (diag(w_t) + a_t b_t^T) + v_t k_t^T,
// y_t = S_t r_t) is affine in the chunk's entry state, because the transition
// diag(w_t) + a_t b_t^T does not depend on S:
//     S_out = S_in M_c + E_c,   y_t = S_in q_t + (terms without S_in).
// The chunked forward builds [M_c^T; Q_c] (Q_c's rows are the q_t) for its own
// state round; its checkpoint pass exports it per chunk (kMqChunkVec, bf16
// hi / lo images).  The adjoint of the map is then one product per chunk:
//     dS_in = dS_out M_c^T + dY_c^T Q_c,   dS_out(c - 1) = dS_in(c),
// i.e. [dS_in] (64 x 64) = [dS_out | dY_c^T] (64 x 96) . [M_c^T; Q_c] (96 x 64).
// This replaces the per-token sweep of the state gradient (bwd_dstate_kernel)
// when the transitions are at hand: the chain takes one tensor-core step per
// chunk instead of 32 CUDA-core steps.
//
// One CTA per (b, h) walks its chunks from the last to the first; 8 warps
// read the result and prepare the next step, thread 0 issues the MMAs
// (M = 64, N = 64: dS_out hi / lo split, three passes over K = 64; dY exact
// in bf16, two passes over K = 32), and its wait for their completion is
// bounded.  The next two chunks' [M^T; Q] and dY tiles are staged by cp.async
// (two stages) while the current step runs.
#include <algorithm>

#include "umma.cuh"

namespace wkv7 {

namespace dchain {

constexpr int L = 32;
constexpr int NT = 256;
constexpr uint32_t TMEM_COLS = 64;
constexpr uint32_t MQ_BYTES = kMqChunkVec * 16;        // hi image, then lo image
constexpr uint32_t MQ0 = 0;                            // [2 stages] transition images
constexpr uint32_t DY0 = 2 * MQ_BYTES;                 // [2 stages] dY [32 t][64 i], core-matrix layout
constexpr uint32_t DY_BYTES = L * kN * 2;
constexpr uint32_t D_HI = DY0 + 2 * DY_BYTES;          // dS_out [64 i][64 m], hi and lo
constexpr uint32_t D_LO = D_HI + kN * kN * 2;
constexpr uint32_t BAR = D_LO + kN * kN * 2;           // one mbarrier: the step's MMAs are done
constexpr uint32_t TMEM_SLOT = BAR + 8;
constexpr uint32_t FLAG = BAR + 12;
constexpr uint32_t SMEM_BYTES = BAR + 64;
constexpr long long kDrainCycles = 200000000LL;

}  // namespace dchain

__global__ void __launch_bounds__(dchain::NT)
bwd_dchain_kernel(int T, int H, const __nv_bfloat16 *__restrict__ dy, const uint4 *__restrict__ mq,
                  const float *__restrict__ dsT, float *__restrict__ dS_out, float *__restrict__ ds0,
                  long long wait_limit) {
    using namespace dchain;
    using namespace umma;
    extern __shared__ __align__(1024) unsigned char sm[];
    const uint32_t sbase = smem_u32(sm);
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int head = blockIdx.x, bb = head / H, h = head % H;
    const int nck = (T + L - 1) / L;
    const size_t tok_stride = (size_t)H * kN;
    const size_t base = ((size_t)bb * T * H + h) * kN;
    const size_t hoff = (size_t)head * kN * kN;
    volatile uint32_t *abort_flag = reinterpret_cast<volatile uint32_t *>(sm + FLAG);
    auto mq_stage = [&](int s) { return MQ0 + (uint32_t)s * MQ_BYTES; };
    auto dy_stage = [&](int s) { return DY0 + (uint32_t)s * DY_BYTES; };

    // [M^T; Q] and dY of chunk c into a stage (one cp.async group per call,
    // empty when c < 0); dY rows past the end of the sequence are zeros
    auto issue = [&](int c, int s) {
        if (c >= 0) {
            const uint4 *src = mq + ((size_t)head * nck + c) * kMqChunkVec;
            for (int x = tid; x < kMqChunkVec; x += NT) cp_async16(sm + mq_stage(s) + 16 * x, src + x);
            const int t = tid >> 3, ch = tid & 7;
            unsigned char *dst = sm + dy_stage(s) + cm_off(t, 8 * ch, kN);
            if (c * L + t < T) cp_async16(dst, dy + base + (size_t)(c * L + t) * tok_stride + 8 * ch);
            else *reinterpret_cast<uint4 *>(dst) = make_uint4(0, 0, 0, 0);
        }
        cp_async_commit();
    };

    if (tid == 0) {
        mbar_init(sbase + BAR, 1);
        *abort_flag = 0;
    }
    if (warp == 0) tmem_alloc(sbase + TMEM_SLOT, TMEM_COLS);
    issue(nck - 1, 0);
    issue(nck - 2, 1);
    {   // dS_out of the last chunk = dsT (zeros when null): to dS_out and to the A operand
        const int i = tid >> 2, c0 = 16 * (tid & 3);
        float x[16];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
            const float4 d = dsT ? load4(dsT + hoff + (size_t)i * kN + c0 + 4 * u) : make_float4(0.f, 0.f, 0.f, 0.f);
            x[4 * u] = d.x; x[4 * u + 1] = d.y; x[4 * u + 2] = d.z; x[4 * u + 3] = d.w;
            store4(dS_out + ((size_t)head * nck + nck - 1) * kN * kN + (size_t)i * kN + c0 + 4 * u, d);
        }
        store8_split(sm + D_HI, sm + D_LO, cm_off(i, c0, kN), x);
        store8_split(sm + D_HI, sm + D_LO, cm_off(i, c0 + 8, kN), x + 8);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_before_sync();
    __syncthreads();
    fence_after_sync();
    const uint32_t tmem = *reinterpret_cast<volatile uint32_t *>(sm + TMEM_SLOT);

    // dS_out M^T: A = dS_out rows i (K-major, K = m), B = M^T rows m (MN-major, N = j)
    const uint32_t id_d = idesc_bf16(64, 64, 0, 1);
    // dY^T Q: A = dY rows t (MN-major: K = t, M = i), exact; B = Q rows t (MN-major)
    const uint32_t id_y = idesc_bf16(64, 64, 1, 1);
    const int q4 = warp & 3, half = warp >> 2;        // TMEM lane quadrant, 32-column half
    const int i = 16 * q4 + (lane & 15);              // result row (M = 64 layout: lanes 0-15 of a quadrant)
    int last_it = -1;

    for (int it = 0; it < nck; ++it) {
        const int c = nck - 1 - it, s = it & 1;
        cp_async_wait<1>();                           // chunk c's stage (the next one may still be in flight)
        fence_smem_to_async();
        fence_before_sync();
        __syncthreads();
        if (tid == 0) {
            fence_after_sync();
            if (*abort_flag == 0u) {
                const OpD dA = opd_k(sbase + D_HI, sbase + D_LO, kN);
                const OpD mB = opd_mn(sbase + mq_stage(s), sbase + mq_stage(s) + MQ_BYTES / 2, kN);
                const OpD yA = opd_mn(sbase + dy_stage(s), 0, kN);
                const uint32_t qoff = cm_off(kN, 0, kN);      // row 64 of the image: Q
                const OpD qB = opd_mn(sbase + mq_stage(s) + qoff, sbase + mq_stage(s) + MQ_BYTES / 2 + qoff, kN);
                gemm_split_d(tmem, dA, mB, id_d, kN / 16, false);
                gemm_split_d(tmem, yA, qB, id_y, L / 16, true);
                commit(sbase + BAR);
                last_it = it;
                if (!mbar_spin(sbase + BAR, (uint32_t)it & 1u, wait_limit)) *abort_flag = 1;
            }
            fence_before_sync();
        }
        __syncthreads();
        fence_after_sync();
        issue(c - 2, s);                              // the stage is free again
        uint32_t r0[16], r1[16];
        tmem_ld16_nowait(tmem + ((uint32_t)(32 * q4) << 16) + 32u * (uint32_t)half, r0);
        tmem_ld16_nowait(tmem + ((uint32_t)(32 * q4) << 16) + 32u * (uint32_t)half + 16, r1);
        tmem_wait();
        if (lane < 16) {
            float x[32];
#pragma unroll
            for (int e = 0; e < 16; ++e) {
                x[e] = __uint_as_float(r0[e]);
                x[16 + e] = __uint_as_float(r1[e]);
            }
            float *dst = (c > 0 ? dS_out + ((size_t)head * nck + c - 1) * kN * kN : ds0 + hoff) + (size_t)i * kN +
                         32 * half;
#pragma unroll
            for (int u = 0; u < 8; ++u) store4(dst + 4 * u, make_float4(x[4 * u], x[4 * u + 1], x[4 * u + 2], x[4 * u + 3]));
            if (c > 0) {
#pragma unroll
                for (int u = 0; u < 4; ++u) store8_split(sm + D_HI, sm + D_LO, cm_off(i, 32 * half + 8 * u, kN), x + 8 * u);
            }
        }
    }
    cp_async_wait<0>();

    // ---- tear-down ----
    fence_before_sync();
    __syncthreads();
    if (*abort_flag) {
        // the wait gave up: report it and let the committed MMAs finish before TMEM is released
        if (tid == 0) {
            raise_status(WKV7_ERR_TIMEOUT);
            if (last_it >= 0) mbar_wait(sbase + BAR, (uint32_t)last_it & 1u, kDrainCycles);
        }
        __syncthreads();
    }
    fence_after_sync();
    if (warp == 0) tmem_dealloc(tmem, TMEM_COLS);
}

// dS_out at every chunk end and ds0 by the transition chain (bf16 dy; mq as
// the chunked forward's checkpoint pass exported it).
cudaError_t bwd_dchain(int B, int T, int H, const void *dy, const uint4 *mq, const float *dsT, float *dS_out,
                       float *ds0, long long wait_limit, cudaStream_t st) {
    static_assert(dchain::SMEM_BYTES <= 227 * 1024, "shared memory");
    auto kern = bwd_dchain_kernel;
    cudaError_t e =
        cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)dchain::SMEM_BYTES);
    if (e != cudaSuccess) return e;
    kern<<<(unsigned)((size_t)B * H), dchain::NT, dchain::SMEM_BYTES, st>>>(
        T, H, static_cast<const __nv_bfloat16 *>(dy), mq, dsT, dS_out, ds0, wait_limit);
    return cudaGetLastError();
}

// Bytes of the transition images of every chunk.
size_t bwd_mq_bytes(int B, int T, int H) {
    const size_t nck = ((size_t)T + dchain::L - 1) / dchain::L;
    return (size_t)B * H * nck * kMqChunkVec * 16;
}

// Estimated time (ns) of the chain: a step of about 0.7 us per chunk and CTA
// (three CTAs fit on an SM), or the memory traffic (the transition image and
// dY read, dS written: 44 KiB per chunk) at 6 TB/s, whichever is longer.
double bwd_dchain_ns(int B, int T, int H, int sms) {
    const long long heads = (long long)B * H, nck = (T + dchain::L - 1) / dchain::L;
    if (sms <= 0) sms = 148;
    const long long waves = (heads + 3LL * sms - 1) / (3LL * sms);
    const double lat = (double)waves * (double)nck * 700.0;
    const double mem = (double)heads * (double)nck * 45056.0 / 6000.0;
    return std::max(lat, mem);
}

}  // namespace wkv7
