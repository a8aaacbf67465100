// w4_actorder.cuh -- act-order (GPTQ g_idx) weights with contiguous groups.
//
// An act-order vector g_idx assigns input channel k to group g_idx[k] (per-group scale
// and zero point: "The Ultimate Guide to Quantized LLMs: GPTQ" and "Understanding
// Quantized Model Compression"), so a group's channels are scattered along K.  When every
// group holds exactly group_size channels, ordering the channels by group (stably) makes
// the groups contiguous runs again: with perm[k'] = the k'-th channel in that order,
//   Y[m,n] = sum_k X'[m,k] What[n,k] = sum_k' X'[m,perm[k']] What[n,perm[k']],
// and What[n,perm[k']] belongs to group k' / group_size.  The packer stores the codes in
// the k' order (an ordinary contiguous-group matrix), and the GEMM gathers the activation
// columns through perm once per call; everything in between is the contiguous-group path.
#pragma once
#include "w4_common.cuh"

namespace w4a {

// perm = channels sorted by g_idx, ties in channel order; one warp walks K in order, 32
// channels at a time: peers with the same group take consecutive slots after the slots
// earlier chunks used.  A group with more or fewer than group_size channels, or an entry
// outside [0, G), is reported through the device error word (W4_DEVERR_GIDX); perm is then
// incomplete.  Shared memory: G counters.
__global__ void actorder_perm_kernel(const int32_t* __restrict__ g_idx, int K, int group_size, int G,
                                     int32_t* __restrict__ perm) {
    extern __shared__ int cnt[];
    const int lane = threadIdx.x;
    for (int i = lane; i < G; i += 32) cnt[i] = 0;
    __syncwarp();
    bool bad = false;
    for (int k0 = 0; k0 < K; k0 += 32) {
        const int k = k0 + lane;
        int g = k < K ? __ldg(g_idx + k) : -1;
        if (k < K && (g < 0 || g >= G)) {
            bad = true;
            g = -1;
        }
        const unsigned peers = __match_any_sync(0xffffffffu, g);
        if (g >= 0) {
            const int slot = cnt[g] + __popc(peers & ((1u << lane) - 1u));
            if (slot < group_size) perm[(size_t)g * group_size + slot] = k;
            else bad = true;
        }
        __syncwarp();
        // the highest lane of each group of peers advances the group's counter
        if (g >= 0 && (peers >> lane) == 1u) cnt[g] += __popc(peers);
        __syncwarp();
    }
    for (int i = lane; i < G; i += 32)
        if (cnt[i] != group_size) bad = true;
    if (bad) atomicOr(&g_w4_error_word, W4_DEVERR_GIDX);
}

// Xp[m,k'] = X[m,perm[k']] * s_inv[perm[k']] rounded to the activation type (s_inv NULL:
// the plain gather); one thread per 8 consecutive k'.  An entry of perm outside [0, K) is
// reported through the device error word and reads channel 0.
template <bool BF16>
__global__ void gather_acts_kernel(const void* __restrict__ X, const int32_t* __restrict__ perm,
                                   const float* __restrict__ s_inv, void* __restrict__ Xp, int M, int K) {
    const unsigned short* x = reinterpret_cast<const unsigned short*>(X);
    const int cpt = K / 8;
    const size_t chunks = (size_t)M * cpt;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < chunks;
         i += (size_t)gridDim.x * blockDim.x) {
        const int m = (int)(i / cpt), c = (int)(i % cpt);
        const int4 p0 = __ldg(reinterpret_cast<const int4*>(perm) + 2 * c);
        const int4 p1 = __ldg(reinterpret_cast<const int4*>(perm) + 2 * c + 1);
        int src[8] = {p0.x, p0.y, p0.z, p0.w, p1.x, p1.y, p1.z, p1.w};
        float v[8];
#pragma unroll
        for (int j = 0; j < 8; ++j) {
            if (src[j] < 0 || src[j] >= K) {
                atomicOr(&g_w4_error_word, W4_DEVERR_GIDX);
                src[j] = 0;
            }
            const unsigned short b = x[(size_t)m * K + src[j]];
            float f;
            if constexpr (BF16) f = __bfloat162float(__ushort_as_bfloat16(b));
            else f = __half2float(__ushort_as_half(b));
            v[j] = s_inv ? __fmul_rn(f, __ldg(s_inv + src[j])) : f;
        }
        uint4 out;
        out.x = pack2<BF16>(v[0], v[1]);
        out.y = pack2<BF16>(v[2], v[3]);
        out.z = pack2<BF16>(v[4], v[5]);
        out.w = pack2<BF16>(v[6], v[7]);
        reinterpret_cast<uint4*>(Xp)[i] = out;
    }
}

}  // namespace w4a
