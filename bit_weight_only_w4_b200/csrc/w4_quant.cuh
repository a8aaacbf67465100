// w4_quant.cuh -- AWQ weight scaling + group-wise RTN INT4 quantisation + packing
// into the device layout, and the device -> canonical unpack used by tests.
//
// Method: "Quantization Paradigms for Edge Inference: AWQ, GPTQ, and FP8 Matrix Cores",
// sec. 3, eq. 1 (W' = W diag(s)); "The Ultimate Guide to Quantized LLMs: GPTQ",
// "Understanding Quantized Model Compression" (per-group scale and zero point);
// edgesiliconlab.com article on AWQ vs GPTQ, "What Is the Core Difference ..." (round to
// nearest) and "Kernel Execution ...", item 3 (two 4-bit codes per byte).
#pragma once
#include "w4_common.cuh"

namespace w4q {

constexpr int kThreads = 256;
constexpr int kRows = 16;  // one row tile of the device layout

struct QuantParams {
    const void* W;          // [N,K] fp16 or bf16
    const float* s;         // [K] or null
    const int32_t* g_idx;   // [K] or null
    const int32_t* perm;    // [K] or null: column k of the packed matrix is channel perm[k]
    uint32_t* qweight;      // [N*K/8] device layout
    __half* scales;         // [G,N]
    __half* zeros;          // [G,N] or null (symmetric)
    int N, K, group_size, G, symmetric;
};

// Order-preserving map of floats onto signed ints (for shared-memory atomic min/max).
W4_DEV int f2ord(float f) {
    int i = __float_as_int(f);
    return i >= 0 ? i : (i ^ 0x7FFFFFFF);
}
W4_DEV float ord2f(int i) { return __int_as_float(i >= 0 ? i : (i ^ 0x7FFFFFFF)); }

template <bool BF16W>
W4_DEV float load_w(const void* W, size_t idx) {
    if constexpr (BF16W) return __bfloat162float(reinterpret_cast<const __nv_bfloat16*>(W)[idx]);
    else return __half2float(reinterpret_cast<const __half*>(W)[idx]);
}

// W'[n,k] = fp32(W) * s[k]: exactly one fp32 rounding (no contraction).  With perm,
// column k is channel perm[k] (an entry outside [0, K) is reported and reads channel 0).
template <bool BF16W>
W4_DEV float scaled_w(const QuantParams& p, int n, int k) {
    int src = k;
    if (p.perm) {
        src = __ldg(p.perm + k);
        if (src < 0 || src >= p.K) {
            atomicOr(&g_w4_error_word, W4_DEVERR_GIDX);
            src = 0;
        }
    }
    float w = load_w<BF16W>(p.W, (size_t)n * p.K + src);
    return p.s ? __fmul_rn(w, __ldg(p.s + src)) : w;
}

W4_DEV int group_of(const QuantParams& p, int k) {
    if (!p.g_idx) return k / p.group_size;
    int g = __ldg(p.g_idx + k);
    if (g < 0 || g >= p.G) {
        atomicOr(&g_w4_error_word, W4_DEVERR_GIDX);
        return -1;
    }
    return g;
}

// One CTA per tile of 16 output rows.  Shared memory: two ordered-int tables
// [G][16] holding each (group, row)'s min and max of W', later overwritten by the
// fp32 scale and zero point.
template <bool BF16W>
__global__ void __launch_bounds__(kThreads) quantize_pack_kernel(QuantParams p) {
    extern __shared__ int smem_q[];
    int* tmin = smem_q;
    int* tmax = smem_q + p.G * kRows;
    const int tid = threadIdx.x;
    const int n0 = blockIdx.x * kRows;
    const int lane = tid & 31;

    for (int i = tid; i < p.G * kRows; i += kThreads) {
        tmin[i] = f2ord(__int_as_float(0x7F800000));   // +inf
        tmax[i] = f2ord(__int_as_float(0xFF800000));   // -inf
    }
    __syncthreads();

    // pass 1: range of every (group, row)
    if (!p.g_idx) {
        // groups are runs of >= 32 aligned channels: a warp's 32 consecutive channels
        // share one group, so reduce in the warp first
        for (int k = tid; k < p.K; k += kThreads) {
            const int g = k / p.group_size;
            for (int r = 0; r < kRows; ++r) {
                const int v = f2ord(scaled_w<BF16W>(p, n0 + r, k));
                const int vmin = __reduce_min_sync(0xFFFFFFFFu, v);
                const int vmax = __reduce_max_sync(0xFFFFFFFFu, v);
                if (lane == 0) {
                    atomicMin(&tmin[g * kRows + r], vmin);
                    atomicMax(&tmax[g * kRows + r], vmax);
                }
            }
        }
    } else {
        for (int k = tid; k < p.K; k += kThreads) {
            const int g = group_of(p, k);
            if (g < 0) continue;
            for (int r = 0; r < kRows; ++r) {
                const int v = f2ord(scaled_w<BF16W>(p, n0 + r, k));
                atomicMin(&tmin[g * kRows + r], v);
                atomicMax(&tmax[g * kRows + r], v);
            }
        }
    }
    __syncthreads();

    // pass 2: scale (rounded to fp16) and zero point per (group, row)
    const float min_scale = 6.103515625e-05f;  // 2^-14, smallest normal fp16
    for (int i = tid; i < p.G * kRows; i += kThreads) {
        const int g = i / kRows, r = i % kRows;
        const float mn = ord2f(tmin[i]), mx = ord2f(tmax[i]);
        float s_f;
        if (p.symmetric) s_f = __fdiv_rn(fmaxf(-mn, mx), 7.0f);
        else s_f = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
        s_f = fmaxf(s_f, min_scale);
        const __half s16 = __float2half_rn(s_f);
        const float sc = __half2float(s16);
        float z = 8.0f;
        if (!p.symmetric) z = fminf(fmaxf(rintf(__fdiv_rn(-mn, sc)), 0.0f), 15.0f);
        p.scales[(size_t)g * p.N + n0 + r] = s16;
        if (p.zeros) p.zeros[(size_t)g * p.N + n0 + r] = __float2half_rn(z);
        tmin[i] = __float_as_int(sc);
        tmax[i] = __float_as_int(z);
    }
    __syncthreads();

    // pass 3: quantise and pack, one device-layout word per thread iteration.  Row tile
    // t = blockIdx.x is tile tt of band b; its atom for column block a is atom
    // 8*(K/64)*b + a*Tb + tt (Tb = tiles in the band).
    const int KA = p.K / 64;
    const int words = KA * 128;
    const int T = p.N / 16, b = blockIdx.x >> 3, tt = blockIdx.x & 7;
    const int Tb = min(8, T - 8 * b);
    uint32_t* out = p.qweight + (size_t)128 * ((size_t)8 * KA * b + tt);
    for (int wi = tid; wi < words; wi += kThreads) {
        const int a = wi >> 7, inw = wi & 127;
        const int L = inw >> 2, j = inw & 3;
        const int r0 = L >> 2, c = 2 * (L & 3), kb = 64 * a + 16 * j;
        // (row offset, column offset) of nibbles 0..7
        const int rsel[8] = {0, 8, 0, 8, 0, 8, 0, 8};
        const int csel[8] = {0, 0, 8, 8, 1, 1, 9, 9};
        uint32_t word = 0;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
            const int r = r0 + rsel[i];
            const int k = kb + c + csel[i];
            const int g = group_of(p, k);
            uint32_t qv = 0;
            if (g >= 0) {
                const float sc = __int_as_float(tmin[g * kRows + r]);
                const float z = __int_as_float(tmax[g * kRows + r]);
                const float t = rintf(__fdiv_rn(scaled_w<BF16W>(p, n0 + r, k), sc));
                qv = (uint32_t)fminf(fmaxf(t + z, 0.0f), 15.0f);
            }
            word |= qv << (4 * i);
        }
        out[(size_t)128 * a * Tb + inw] = word;
    }
}

// Device layout -> canonical layout (uint32 [N, K/8], nibble j of word i = q[n][8i+j]):
// code (n, k) sits in atom 8*(K/64)*b + a*Tb + tt of band b = n/128 (tile tt = (n/16)%8,
// column block a = k/64), word 4L + j with L = 4*(n%8) + (k%8)/2, j = (k%64)/16, nibble
// ((n%16)>=8) + 2*((k%16)>=8) + 4*(k%2).
__global__ void unpack_canonical_kernel(const uint32_t* __restrict__ qd, int N, int K,
                                        uint32_t* __restrict__ qc) {
    const int KW = K / 8, KA = K / 64;
    const size_t total = (size_t)N * KW;
    for (size_t idx = blockIdx.x * (size_t)blockDim.x + threadIdx.x; idx < total;
         idx += (size_t)gridDim.x * blockDim.x) {
        const int n = (int)(idx / KW), i = (int)(idx % KW);
        const int t = n >> 4, rr = n & 15, half = rr >> 3, rg = rr & 7;
        const int b = t >> 3, tt = t & 7, Tb = min(8, N / 16 - 8 * b);
        uint32_t out = 0;
        for (int jn = 0; jn < 8; ++jn) {
            const int k = 8 * i + jn;
            const int a = k >> 6, kk = k & 63, j = kk >> 4, cc = kk & 15;
            const int hi8 = cc >> 3, odd = cc & 1, cpair = (cc & 7) >> 1;
            const int L = 4 * rg + cpair;
            const int nib = half + 2 * hi8 + 4 * odd;
            const uint32_t w = qd[(size_t)128 * ((size_t)8 * KA * b + (size_t)a * Tb + tt) + 4 * L + j];
            out |= ((w >> (4 * nib)) & 0xFu) << (4 * jn);
        }
        qc[idx] = out;
    }
}

}  // namespace w4q
