// w4_fp4.cuh -- block-scaled 4-bit floating-point weights (NVFP4, MXFP4): quantisation
// and packing into the device layout, and the element decode the GEMM kernels use.
//
// "Production Quantization: AWQ, GPTQ, GGUF K-quants, FP8, MXFP4/NVFP4", section
// "MXFP4 / NVFP4": 4-bit floating-point weights with a scale per block, the format
// Blackwell's tensor cores run natively.  The encodings follow the formats' published
// definitions:
//   element  E2M1 (sign, 2 exponent bits, 1 mantissa bit): 0, 0.5, 1, 1.5, 2, 3, 4, 6;
//   NVFP4    blocks of 16 along K, an E4M3 block scale, one fp32 tensor scale
//              gs = amax / (6 * 448) (1 for an all-zero tensor),
//              sb = E4M3(blockmax / 6 / gs),  q = E2M1(w / (E4M3(sb) * gs));
//   MXFP4    blocks of 32, a power-of-two block scale 2^e stored as e + 127 (E8M0),
//              e = floor(log2 blockmax) - 2,   q = E2M1(w / 2^e).
// Every conversion rounds to nearest, ties to even, and saturates finite values at the
// largest magnitude (the hardware conversions with .satfinite); the sign of an element
// is the sign of its input, also when it rounds to zero.
//
// The codes take the places of the INT4 codes in the device layout (w4a16.h), so the GEMM
// kernels stage them exactly like INT4 weights.  Block scales are bytes [K/B, N]
// (B = 16 or 32), block-row-major like the INT4 scales.
#pragma once
#include "w4_common.cuh"

namespace w4f {

enum : int { kNvfp4 = 0, kMxfp4 = 1 };

template <int FMT>
struct Fmt {
    static constexpr int block = FMT == kNvfp4 ? 16 : 32;
};

constexpr int kThreads = 256;
constexpr int kRows = 16;  // one row tile of the device layout

// ---------------------------------------------------------------- element conversions
// E2M1 code of x: the magnitude rounded to nearest-even and saturated by the hardware
// conversion, the sign taken from x.
W4_DEV uint32_t f32_to_e2m1(float x) {
    uint32_t b;
    asm("{\n\t.reg .b8 t;\n\tcvt.rn.satfinite.e2m1x2.f32 t, %1, %1;\n\tcvt.u32.u8 %0, t;\n\t}"
        : "=r"(b)
        : "f"(fabsf(x)));
    return (b & 7u) | ((__float_as_uint(x) >> 28) & 8u);
}

// E4M3 byte of a non-negative x (round to nearest-even, saturating at 448).
W4_DEV uint32_t f32_to_e4m3(float x) {
    uint32_t h;
    asm("{\n\t.reg .b16 t;\n\tcvt.rn.satfinite.e4m3x2.f32 t, %1, %1;\n\tcvt.u32.u16 %0, t;\n\t}"
        : "=r"(h)
        : "f"(x));
    return h & 0xFFu;
}

// Two E2M1 codes (the low and high nibble of a byte) -> two fp16 values, exactly.
W4_DEV uint32_t e2m1x2_to_h2(uint32_t byte) {
    uint32_t d;
    asm("{\n\t.reg .b8 t;\n\tcvt.u8.u32 t, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, t;\n\t}" : "=r"(d) : "r"(byte));
    return d;
}

// Two E4M3 bytes (low, high byte of a 16-bit value) -> two fp16 values, exactly.
W4_DEV uint32_t e4m3x2_to_h2(uint32_t two) {
    uint32_t d;
    asm("{\n\t.reg .b16 t;\n\tcvt.u16.u32 t, %1;\n\tcvt.rn.f16x2.e4m3x2 %0, t;\n\t}" : "=r"(d) : "r"(two));
    return d;
}

// (both bytes of the pair are b, so the result does not depend on the pair's order)
W4_DEV float e4m3_to_f32(uint32_t b) {
    b &= 0xFFu;
    return __low2float(u32_as_h2(e4m3x2_to_h2(b | (b << 8))));
}

// One device-layout word -> the four A-operand registers of a 16x16 MMA slice (a[0] =
// row r0 cols c,c+1; a[1] = row r1 cols c,c+1; a[2] = row r0 cols c+8,c+9; a[3] = row r1
// cols c+8,c+9), every element the exact fp16 value of its E2M1 code.  Nibbles i and
// i+4 of the word are a register's two columns, so one conversion each takes the bytes
// (n0|n4), (n2|n6) of the word and (n1|n5), (n3|n7) of the word shifted by 4 (the byte's
// low nibble is the register's first column).
W4_DEV void unpack_fp4(uint32_t w, uint32_t (&a)[4]) {
    const uint32_t zx = (w & 0x0F0Fu) | ((w >> 12) & 0xF0F0u);
    const uint32_t zy = ((w >> 4) & 0x0F0Fu) | ((w >> 16) & 0xF0F0u);
    a[0] = e2m1x2_to_h2(zx & 0xFFu);
    a[1] = e2m1x2_to_h2(zy & 0xFFu);
    a[2] = e2m1x2_to_h2((zx >> 8) & 0xFFu);
    a[3] = e2m1x2_to_h2((zy >> 8) & 0xFFu);
}

// 2^e for e in [-126, 127] (exact; fp32 bit pattern).
W4_DEV float exp2i(int e) { return __int_as_float((e + 127) << 23); }

// ---------------------------------------------------------------- quantisation
struct Fp4Params {
    const void* W;          // [N,K] fp16 or bf16
    uint32_t* qweight;      // [N*K/8] device layout
    uint8_t* bscale;        // [K/B, N]
    float* tscale;          // NVFP4: the tensor amax on entry to the packing kernel, gs after
    int N, K;
};

template <bool BF16W>
W4_DEV float load_w(const void* W, size_t idx) {
    if constexpr (BF16W) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(W)[idx]);
    else return __half2float(reinterpret_cast<const __half*>(W)[idx]);
}

// NVFP4, step 1: amax over the tensor (|w| as ordered bits; *tscale zeroed before).
template <bool BF16W>
__global__ void amax_kernel(const void* W, size_t n, float* amax) {
    float m = 0.0f;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        m = fmaxf(m, fabsf(load_w<BF16W>(W, i)));
    m = __uint_as_float(__reduce_max_sync(0xFFFFFFFFu, __float_as_uint(m)));
    if ((threadIdx.x & 31) == 0 && m > 0.0f) atomicMax(reinterpret_cast<unsigned int*>(amax), __float_as_uint(m));
}

W4_DEV float tensor_scale_of(float amax) { return amax > 0.0f ? __fdiv_rn(amax, 2688.0f) : 1.0f; }

// NVFP4, step 3: the tensor scale replaces the amax.
__global__ void finish_tscale_kernel(float* tscale) { *tscale = tensor_scale_of(*tscale); }

// Step 2 (both formats): one CTA per tile of 16 output rows.  Pass 1: each (block, row)'s
// scale byte, to global memory and to shared memory [K/B][16]; pass 2: the codes, one
// device-layout word per thread iteration (the placement of the INT4 packer).
template <int FMT, bool BF16W>
__global__ void __launch_bounds__(kThreads) fp4_pack_kernel(Fp4Params p) {
    constexpr int B = Fmt<FMT>::block;
    extern __shared__ unsigned char smem_f[];
    const int tid = threadIdx.x;
    const int n0 = blockIdx.x * kRows;
    const int nb = p.K / B;
    const float gs = FMT == kNvfp4 ? tensor_scale_of(*p.tscale) : 1.0f;

    for (int i = tid; i < nb * kRows; i += kThreads) {
        const int b = i / kRows, r = i % kRows;
        const size_t base = (size_t)(n0 + r) * p.K + (size_t)b * B;
        float bmax = 0.0f;
        for (int k = 0; k < B; ++k) bmax = fmaxf(bmax, fabsf(load_w<BF16W>(p.W, base + k)));
        uint32_t byte;
        if constexpr (FMT == kNvfp4) {
            byte = f32_to_e4m3(__fdiv_rn(__fdiv_rn(bmax, 6.0f), gs));
        } else {
            const int e = bmax > 0.0f ? max(ilogbf(bmax) - 2, -127) : -127;
            byte = (uint32_t)(e + 127);
        }
        smem_f[i] = (unsigned char)byte;
        p.bscale[(size_t)b * p.N + n0 + r] = (uint8_t)byte;
    }
    __syncthreads();

    const int KA = p.K / 64;
    const int words = KA * 128;
    const int T = p.N / 16, band = blockIdx.x >> 3, tt = blockIdx.x & 7;
    const int Tb = min(8, T - 8 * band);
    uint32_t* out = p.qweight + (size_t)128 * ((size_t)8 * KA * band + tt);
    for (int wi = tid; wi < words; wi += kThreads) {
        const int a = wi >> 7, inw = wi & 127;
        const int L = inw >> 2, j = inw & 3;
        const int r0 = L >> 2, c = 2 * (L & 3), kb = 64 * a + 16 * j;
        const int rsel[8] = {0, 8, 0, 8, 0, 8, 0, 8};
        const int csel[8] = {0, 0, 8, 8, 1, 1, 9, 9};
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = r0 + rsel[i];
            const int k = kb + c + csel[i];
            const uint32_t byte = smem_f[(k / B) * kRows + r];
            const float w = load_w<BF16W>(p.W, (size_t)(n0 + r) * p.K + k);
            uint32_t q;
            if constexpr (FMT == kNvfp4) {
                const float sd = __fmul_rn(e4m3_to_f32(byte), gs);
                q = sd > 0.0f ? f32_to_e2m1(__fdiv_rn(w, sd)) : 0u;
            } else {
                // w * 2^-e is exact (|w| / 2^e < 8 and 2^-e <= 2^127)
                q = f32_to_e2m1(__fmul_rn(w, exp2i(127 - (int)byte)));
            }
            word |= q << (4 * i);
        }
        out[(size_t)128 * a * Tb + inw] = word;
    }
}

}  // namespace w4f
