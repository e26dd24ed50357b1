// Thin helpers around the sm_100a tensor-core instructions (tcgen05) and
// mbarriers used by the chunked forward.  Operands live in shared memory in the
// no-swizzle "core matrix" layout: 8 rows x 16 bytes per 128-byte core matrix.
//
// A tile stored with rows x cols (cols contiguous inside each core matrix) can
// be presented to the MMA either
//   * K-major  (rows = M or N, cols = K):  LBO = 128 B, SBO = (cols/8) * 128 B
//   * MN-major (cols = M or N, rows = K):  LBO = (cols/8) * 128 B, SBO = 128 B
// i.e. one buffer serves a matrix and its transpose.
#pragma once

#include <stdint.h>

#include "common.cuh"

namespace wkv7 {
namespace umma {

// byte offset of element (r, c) of a rows x cols bf16 tile in core-matrix layout
__device__ __forceinline__ uint32_t cm_off(int r, int c, int cols) {
    return (uint32_t)((((r >> 3) * (cols >> 3) + (c >> 3)) << 7) + ((r & 7) << 4) + ((c & 7) << 1));
}

// shared-memory matrix descriptor (SWIZZLE_NONE, sm_100 version bits)
__device__ __forceinline__ uint64_t sdesc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
           ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | ((uint64_t)1 << 46);
}

// instruction descriptor: bf16 x bf16 -> fp32, dense
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, int a_mn, int b_mn) {
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)a_mn << 15) | ((uint32_t)b_mn << 16) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// One operand view: base addresses of the hi / lo bf16 copies, the descriptor
// strides and the byte step between consecutive K=16 slices.  lo == 0 means
// the operand is exact in bf16 (no low part).
struct Op {
    uint32_t hi, lo, lbo, sbo, kstep;
};

// rows x cols tile used K-major (K = cols)
__device__ __forceinline__ Op op_k(uint32_t hi, uint32_t lo, int cols) {
    return Op{hi, lo, 128u, (uint32_t)(cols >> 3) << 7, 256u};
}
// rows x cols tile used MN-major (K = rows, MN = cols)
__device__ __forceinline__ Op op_mn(uint32_t hi, uint32_t lo, int cols) {
    const uint32_t lbo = (uint32_t)(cols >> 3) << 7;
    return Op{hi, lo, lbo, 128u, 2u * lbo};
}

__device__ __forceinline__ void mma(uint32_t d_tmem, uint64_t a, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "l"(a), "l"(b), "r"(idesc), "r"(acc));
}

// D (+)= A * B^T with bf16 hi/lo split operands: hi*hi + hi*lo + lo*hi (the
// lo*lo term, ~2^-18 relative, is dropped; a pass is skipped when one side is
// exact).  Issued by a single thread.
__device__ __forceinline__ void gemm_split(uint32_t d_tmem, const Op &A, const Op &B, uint32_t idesc, int ksteps,
                                           bool accumulate) {
    uint32_t acc = accumulate ? 1u : 0u;
    for (int ks = 0; ks < ksteps; ++ks) {
        mma(d_tmem, sdesc(A.hi + ks * A.kstep, A.lbo, A.sbo), sdesc(B.hi + ks * B.kstep, B.lbo, B.sbo), idesc, acc);
        acc = 1u;
    }
    if (B.lo)
        for (int ks = 0; ks < ksteps; ++ks)
            mma(d_tmem, sdesc(A.hi + ks * A.kstep, A.lbo, A.sbo), sdesc(B.lo + ks * B.kstep, B.lbo, B.sbo), idesc, 1u);
    if (A.lo)
        for (int ks = 0; ks < ksteps; ++ks)
            mma(d_tmem, sdesc(A.lo + ks * A.kstep, A.lbo, A.sbo), sdesc(B.hi + ks * B.kstep, B.lbo, B.sbo), idesc, 1u);
}

// Operand given by full base descriptors (hi copy, lo copy or 0 when the
// operand is exact in bf16) and the start-address step between K=16 slices,
// in 16-byte units.  Shared-memory addresses stay below 256 KB, so stepping
// the 14-bit start field never carries into the other fields.
struct OpD {
    uint64_t hi, lo;
    uint32_t kstep16;
};

__device__ __forceinline__ OpD opd_k(uint32_t hi, uint32_t lo, int cols) {
    return OpD{sdesc(hi, 128u, (uint32_t)(cols >> 3) << 7), lo ? sdesc(lo, 128u, (uint32_t)(cols >> 3) << 7) : 0ull,
               16u};
}
__device__ __forceinline__ OpD opd_mn(uint32_t hi, uint32_t lo, int cols) {
    const uint32_t lbo = (uint32_t)(cols >> 3) << 7;
    return OpD{sdesc(hi, lbo, 128u), lo ? sdesc(lo, lbo, 128u) : 0ull, (2u * lbo) >> 4};
}

__device__ __forceinline__ void gemm_split_d(uint32_t d_tmem, const OpD &A, const OpD &B, uint32_t idesc, int ksteps,
                                             bool accumulate) {
    uint32_t acc = accumulate ? 1u : 0u;
    for (int ks = 0; ks < ksteps; ++ks) {
        mma(d_tmem, A.hi + ks * A.kstep16, B.hi + ks * B.kstep16, idesc, acc);
        acc = 1u;
    }
    if (B.lo)
        for (int ks = 0; ks < ksteps; ++ks) mma(d_tmem, A.hi + ks * A.kstep16, B.lo + ks * B.kstep16, idesc, 1u);
    if (A.lo)
        for (int ks = 0; ks < ksteps; ++ks) mma(d_tmem, A.lo + ks * A.kstep16, B.hi + ks * B.kstep16, idesc, 1u);
}

// D (+)= A * B with A read from tensor memory (M lanes; bf16 pairs packed per
// 32-bit column, the lower half holding the even K index) and B from shared
// memory.  Split passes: Ahi*Bhi + Ahi*Blo + Alo*Bhi; one K=16 step is 8 columns.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b, uint32_t idesc, uint32_t acc) {
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}\n" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b), "r"(idesc), "r"(acc));
}

__device__ __forceinline__ void gemm_split_ts(uint32_t d_tmem, uint32_t a_hi, uint32_t a_lo, const OpD &B,
                                              uint32_t idesc, int ksteps, bool accumulate) {
    uint32_t acc = accumulate ? 1u : 0u;
    for (int ks = 0; ks < ksteps; ++ks) {
        mma_ts(d_tmem, a_hi + 8u * ks, B.hi + ks * B.kstep16, idesc, acc);
        acc = 1u;
    }
    for (int ks = 0; ks < ksteps; ++ks) mma_ts(d_tmem, a_hi + 8u * ks, B.lo + ks * B.kstep16, idesc, 1u);
    for (int ks = 0; ks < ksteps; ++ks) mma_ts(d_tmem, a_lo + 8u * ks, B.hi + ks * B.kstep16, idesc, 1u);
}

__device__ __forceinline__ void commit(uint32_t mbar_saddr) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(mbar_saddr)
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }
// make generic-proxy shared-memory writes visible to the tensor core (async proxy)
__device__ __forceinline__ void fence_smem_to_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t dst_saddr, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_saddr), "r"(ncols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols));
}

// 32 lanes x 16 consecutive 32-bit columns, without waiting (pair with tmem_wait)
__device__ __forceinline__ void tmem_ld16_nowait(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns from registers (thread t -> lane base + t)
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};" ::"r"(
            taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]), "r"(r[8]), "r"(r[9]),
        "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]), "r"(r[15])
        : "memory");
}
// 32 lanes x 8 consecutive 32-bit columns from registers (thread t -> lane base + t)
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
    asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"r"(taddr), "r"(r[0]),
                 "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7])
                 : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

// 32 lanes x 16 consecutive 32-bit columns; thread t of the warp gets lane (base + t)
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float (&v)[16]) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int j = 0; j < 16; ++j) v[j] = __uint_as_float(r[j]);
}

// ---- mbarrier ---------------------------------------------------------------

__device__ __forceinline__ void mbar_init(uint32_t saddr, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(saddr), "r"(count));
}

// Wait for the phase with the given parity to complete.  Gives up after
// `limit_cycles` (returns false) instead of spinning forever.
__device__ __forceinline__ bool mbar_wait(uint32_t saddr, uint32_t parity, long long limit_cycles) {
    const long long t0 = clock64();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(saddr), "r"(parity)
            : "memory");
        if (done) return true;
        if (clock64() - t0 > limit_cycles) return false;
    }
}

// Same, polling with the non-suspending test_wait (prompt wake-up; for a single
// thread that has nothing else to do).
__device__ __forceinline__ bool mbar_spin(uint32_t saddr, uint32_t parity, long long limit_cycles) {
    const long long t0 = clock64();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(saddr), "r"(parity)
            : "memory");
        if (done) return true;
        if (clock64() - t0 > limit_cycles) return false;
    }
}

// test_wait polling that also gives up as soon as *abort (a shared flag set by
// another warp that gave up) becomes nonzero.  The phase must be observed
// within limit_cycles of the start of the wait: a poll that sees it complete
// after the limit still counts as a timeout.
__device__ __forceinline__ bool mbar_spin_abortable(uint32_t saddr, uint32_t parity, long long limit_cycles,
                                                    const volatile uint32_t *abort) {
    const long long t0 = clock64();
    while (true) {
        uint32_t done;
        asm volatile(
            "{\n\t.reg .pred p;\n\tmbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}\n"
            : "=r"(done)
            : "r"(saddr), "r"(parity)
            : "memory");
        if (clock64() - t0 > limit_cycles) return false;
        if (done) return true;
        if (*abort) return false;
    }
}

__device__ __forceinline__ void mbar_arrive(uint32_t saddr) {
    asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(saddr) : "memory");
}

// named barrier among `count` threads (a multiple of 32)
__device__ __forceinline__ void named_sync(uint32_t id, uint32_t count) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(count) : "memory");
}
// arrive at a named barrier without waiting (producer side)
__device__ __forceinline__ void named_arrive(uint32_t id, uint32_t count) {
    asm volatile("bar.arrive %0, %1;" ::"r"(id), "r"(count) : "memory");
}

// ---- bf16 hi/lo split --------------------------------------------------------

// x ~= hi + lo with hi = bf16(x), lo = bf16(x - hi): 16 significant bits.
__device__ __forceinline__ void split2(float x, __nv_bfloat16 &hi, __nv_bfloat16 &lo) {
    hi = __float2bfloat16_rn(x);
    lo = __float2bfloat16_rn(x - __bfloat162float(hi));
}

// store 8 consecutive values (one core-matrix row) as hi and lo 16-byte vectors
// (packed conversions: two values per cvt, the hi part re-expanded by bit ops)
__device__ __forceinline__ void store8_split(unsigned char *hi_base, unsigned char *lo_base, uint32_t off,
                                             const float *x) {
    uint32_t h[4], l[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
        const __nv_bfloat162 hp = __floats2bfloat162_rn(x[2 * q], x[2 * q + 1]);
        const uint32_t hu = *reinterpret_cast<const uint32_t *>(&hp);
        // x - hi for the pair in one packed fma (exact: -1 * hi is exact)
        const float2 rr = __ffma2_rn(make_float2(__uint_as_float(hu << 16), __uint_as_float(hu & 0xffff0000u)),
                                     make_float2(-1.f, -1.f), make_float2(x[2 * q], x[2 * q + 1]));
        const float r0 = rr.x, r1 = rr.y;
        const __nv_bfloat162 lp = __floats2bfloat162_rn(r0, r1);
        h[q] = hu;
        l[q] = *reinterpret_cast<const uint32_t *>(&lp);
    }
    *reinterpret_cast<uint4 *>(hi_base + off) = make_uint4(h[0], h[1], h[2], h[3]);
    if (lo_base) *reinterpret_cast<uint4 *>(lo_base + off) = make_uint4(l[0], l[1], l[2], l[3]);
}

}  // namespace umma
}  // namespace wkv7
