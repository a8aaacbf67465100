// w4_common.cuh -- small sm_100a building blocks shared by the W4A16 kernels:
// mbarriers with bounded waits, TMA bulk / tensor copies, warp-level MMA, INT4 unpack.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define W4_DEV __device__ __forceinline__

// Device error word (bit 0: a bounded wait expired; bit 1: out-of-range g_idx entry).
__device__ unsigned int g_w4_error_word;
// Bound of every wait, in nanoseconds of %globaltimer.
__device__ unsigned long long g_w4_wait_limit_ns = 2000000000ull;

enum : unsigned { W4_DEVERR_TIMEOUT = 1u, W4_DEVERR_GIDX = 2u };

W4_DEV uint32_t smem_u32(const void* p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// The first 1024-byte aligned address of a dynamic shared-memory array, by pointer
// arithmetic on the array itself so that the compiler still knows the result points to
// shared memory (loads through it stay shared-memory loads, not generic ones).
W4_DEV unsigned char* align_smem_1024(unsigned char* raw) {
    return raw + ((1024u - (smem_u32(raw) & 1023u)) & 1023u);
}

W4_DEV uint64_t globaltimer_ns() {
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// ---------------------------------------------------------------- mbarriers
W4_DEV void mbar_init(uint64_t* bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

W4_DEV void fence_mbar_init() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

W4_DEV void mbar_arrive(uint64_t* bar) {
    asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

W4_DEV void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;" ::"r"(
                     smem_u32(bar)),
                 "r"(bytes)
                 : "memory");
}

W4_DEV bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// try_wait that may suspend the thread for up to `ns` nanoseconds while the phase is
// incomplete; the thread resumes when the phase completes.  A waiting warp then takes no
// issue slots from the warps doing work.
W4_DEV bool mbar_try_wait_sleep(uint64_t* bar, uint32_t parity, uint32_t ns) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.acquire.cta.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(ns)
        : "memory");
    return ok != 0;
}

// Wait for the phase with the given parity to complete.  Bounded: after the configured
// limit the device error word records a timeout and false is returned.  Each try suspends
// the warp (up to 20 us) instead of spinning, so waiting warps leave the issue slots to
// the working ones; the clock and the limit (a global load) are only read once a wait has
// lasted a while.
W4_DEV bool mbar_wait(uint64_t* bar, uint32_t parity) {
    if (mbar_try_wait(bar, parity)) return true;
    for (uint32_t i = 0; i < 8; ++i)
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = *(volatile unsigned long long*)&g_w4_wait_limit_ns;
    for (;;) {
        if (mbar_try_wait_sleep(bar, parity, 20000u)) return true;
        if (globaltimer_ns() - t0 > limit) {
            atomicOr(&g_w4_error_word, W4_DEVERR_TIMEOUT);
            return false;
        }
    }
}

// ---------------------------------------------------------------- programmatic dependent launch
// Let the next kernel on the stream (launched with programmatic stream serialization)
// start its prologue while this grid finishes.
W4_DEV void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }
// Wait until the preceding grid has completed and its memory operations are visible.
W4_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

// One lane of a converged warp (the same lane for every caller in the warp).
W4_DEV bool elect_one() {
    uint32_t pred = 0;
    asm volatile(
        "{\n\t.reg .pred P;\n\telect.sync _|P, 0xffffffff;\n\tselp.u32 %0, 1, 0, P;\n\t}"
        : "=r"(pred));
    return pred != 0;
}

// ---------------------------------------------------------------- named barriers
W4_DEV void named_bar_sync(uint32_t id, uint32_t nthreads) {
    asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(nthreads) : "memory");
}

// ---------------------------------------------------------------- TMA copies
// 1-D bulk copy global -> shared, completing `bytes` of transaction on `bar`.
// dst and src 16-byte aligned, bytes a multiple of 16.
W4_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::
            "r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar))
        : "memory");
}

// Same, with an L2 eviction-priority policy (streamed-once data).
W4_DEV void bulk_g2s_hint(void* dst, const void* src, uint32_t bytes, uint64_t* bar,
                          uint64_t policy) {
    asm volatile(
        "cp.async.bulk.shared::cta.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], "
        "[%1], %2, [%3], %4;" ::"r"(smem_u32(dst)),
        "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

W4_DEV uint64_t policy_evict_first() {
    uint64_t p;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}

// 2-D tiled tensor copy global -> shared (box given by the tensor map).
W4_DEV void tma_load_2d(void* dst, const CUtensorMap* map, int32_t c0, int32_t c1,
                        uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cta.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3}], [%4];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(smem_u32(bar))
        : "memory");
}

// 3-D tiled tensor copy global -> shared (box given by the tensor map).
W4_DEV void tma_load_3d(void* dst, const CUtensorMap* map, int32_t c0, int32_t c1, int32_t c2,
                        uint64_t* bar) {
    asm volatile(
        "cp.async.bulk.tensor.3d.shared::cta.global.tile.mbarrier::complete_tx::bytes "
        "[%0], [%1, {%2, %3, %4}], [%5];" ::"r"(smem_u32(dst)),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(c0), "r"(c1), "r"(c2), "r"(smem_u32(bar))
        : "memory");
}

W4_DEV void prefetch_tensormap(const CUtensorMap* map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// Make this thread's generic-proxy shared-memory writes visible to the async proxy
// (TMA, tensor cores).
W4_DEV void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// ---------------------------------------------------------------- warp-level MMA
// D(16x8, fp32) += A(16x16, row) * B(16x8, col); operands fp16 or bf16.
template <bool BF16>
W4_DEV void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (BF16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
            : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
    }
}

// ---------------------------------------------------------------- INT4 unpack
// (x & mask) | bias in one LOP3.
W4_DEV uint32_t and_or(uint32_t x, uint32_t mask, uint32_t bias) {
    uint32_t r;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(r) : "r"(x), "r"(mask), "r"(bias));
    return r;
}

W4_DEV uint32_t h2_as_u32(__half2 h) { return *reinterpret_cast<uint32_t*>(&h); }
W4_DEV __half2 u32_as_h2(uint32_t u) { return *reinterpret_cast<__half2*>(&u); }
W4_DEV uint32_t b2_as_u32(__nv_bfloat162 h) { return *reinterpret_cast<uint32_t*>(&h); }
W4_DEV __nv_bfloat162 u32_as_b2(uint32_t u) { return *reinterpret_cast<__nv_bfloat162*>(&u); }

// Per-row constants for the exact unpack of one packed word.
struct ZeroConsts {
    uint32_t lo0, lo1;  // (bias + z) for the plain nibble pairs of row r0 / r1
    uint32_t hi0, hi1;  // fp16 only: (64 + z) negated, for the x16 nibble pairs
};

// fp16: an fp16 with exponent field 25 (bits 0x6400) has unit spacing on [1024, 2048),
// so OR-ing a nibble q into its low mantissa bits gives exactly 1024 + q; a nibble in
// bits 4..7 gives 1024 + 16 q.  Subtracting (1024 + z), resp. scaling by 1/16 and
// subtracting (64 + z), yields the exact integer q - z.  bf16: exponent 134 (bits 0x4300)
// has unit spacing on [128, 256).

// The constants (bias + z) for the unpack below, straight from the fp16 zero points
// (integers 0..15) of rows r0 / r1, with fp16 arithmetic and byte permutes only (no type
// conversions):
//   s = (1024 + z0, 1024 + z1)   exact in fp16, and its low mantissa nibbles are z0, z1;
//   fp16: lo0 = (1024 + z0) x2, hi1 = (960 - (1024 + z1)) x2 = -(64 + z1) x2;
//   bf16: lo0 = 0x4300 | z0 (x2), lo1 = 0x4300 | z1 (x2)   (128 + z in bf16).
// The symmetric format's implicit zero point is z = 8 (fp16 bits 0x4800).
template <bool BF16>
W4_DEV ZeroConsts zero_consts_h(uint32_t z0_bits, uint32_t z1_bits) {
    const uint32_t zz = __byte_perm(z0_bits, z1_bits, 0x5410);              // (z0, z1)
    const uint32_t s = h2_as_u32(__hadd2(u32_as_h2(zz), u32_as_h2(0x64006400u)));
    ZeroConsts zc;
    if constexpr (!BF16) {
        const uint32_t t = h2_as_u32(__hsub2(u32_as_h2(0x63806380u), u32_as_h2(s)));
        zc.lo0 = __byte_perm(s, 0, 0x1010);
        zc.lo1 = __byte_perm(s, 0, 0x3232);
        zc.hi0 = __byte_perm(t, 0, 0x1010);
        zc.hi1 = __byte_perm(t, 0, 0x3232);
    } else {
        const uint32_t z0 = s & 0xFu, z1 = (s >> 16) & 0xFu;
        zc.lo0 = 0x43004300u | z0 | (z0 << 16);
        zc.lo1 = 0x43004300u | z1 | (z1 << 16);
        zc.hi0 = zc.lo0;
        zc.hi1 = zc.lo1;
    }
    return zc;
}

// Unpack one device-layout word into the four A-operand registers of a 16x16 MMA
// slice: a[0] = row r0 cols c,c+1; a[1] = row r1 cols c,c+1; a[2] = row r0 cols
// c+8,c+9; a[3] = row r1 cols c+8,c+9; every element exactly q - z.
template <bool BF16>
W4_DEV void unpack_word(uint32_t w, const ZeroConsts& zc, uint32_t (&a)[4]) {
    if constexpr (!BF16) {
        const __half2 sixteenth = u32_as_h2(0x2C002C00u);   // (1/16, 1/16) in fp16
        const uint32_t w8 = w >> 8;
        a[0] = h2_as_u32(__hsub2(u32_as_h2(and_or(w, 0x000F000Fu, 0x64006400u)), u32_as_h2(zc.lo0)));
        a[1] = h2_as_u32(__hfma2(u32_as_h2(and_or(w, 0x00F000F0u, 0x64006400u)), sixteenth,
                                 u32_as_h2(zc.hi1)));
        a[2] = h2_as_u32(__hsub2(u32_as_h2(and_or(w8, 0x000F000Fu, 0x64006400u)), u32_as_h2(zc.lo0)));
        a[3] = h2_as_u32(__hfma2(u32_as_h2(and_or(w8, 0x00F000F0u, 0x64006400u)), sixteenth,
                                 u32_as_h2(zc.hi1)));
    } else {
        a[0] = b2_as_u32(__hsub2(u32_as_b2(and_or(w, 0x000F000Fu, 0x43004300u)), u32_as_b2(zc.lo0)));
        a[1] = b2_as_u32(__hsub2(u32_as_b2(and_or(w >> 4, 0x000F000Fu, 0x43004300u)), u32_as_b2(zc.lo1)));
        a[2] = b2_as_u32(__hsub2(u32_as_b2(and_or(w >> 8, 0x000F000Fu, 0x43004300u)), u32_as_b2(zc.lo0)));
        a[3] = b2_as_u32(__hsub2(u32_as_b2(and_or(w >> 12, 0x000F000Fu, 0x43004300u)), u32_as_b2(zc.lo1)));
    }
}

// Convert two fp32 values to a packed pair of the activation type (RNE).
template <bool BF16>
W4_DEV uint32_t pack2(float lo, float hi) {
    if constexpr (BF16) return b2_as_u32(__floats2bfloat162_rn(lo, hi));
    else return h2_as_u32(__floats2half2_rn(lo, hi));
}

template <bool BF16>
W4_DEV float2 unpack2(uint32_t v) {
    if constexpr (BF16) return __bfloat1622float2(u32_as_b2(v));
    else return __half22float2(u32_as_h2(v));
}
