// w4_decode.cuh -- bandwidth-bound W4A16 kernel for small M (decode, M <= 64).
//
// Decode reads every weight once per token and is limited by memory bandwidth
// (edgesiliconlab.com article on AWQ vs GPTQ, "The Mathematics of Memory Bandwidth
// Saturation"); the packed weights are staged global -> shared by asynchronous bulk
// copies into a multi-stage ring so the next tiles load while the current ones are
// unpacked and multiplied ("Kernel Execution: Marlin vs. ExLlamaV2 INT4 GEMM
// Micro-Architecture", items 1-2), and unpacked with AND/OR bit tricks right before the
// tensor-core MMA (item 3).
//
// Work decomposition (B200-specific):
//   atom      = 16 output rows x 64 input channels (512 B of codes); the atoms of one
//               128-row band are stored column block by column block, so up to 4
//               consecutive column blocks of a band (up to 16 KB) are one contiguous copy;
//   stream-K  = all (band, column block) atoms of the layer are split into equal
//               contiguous ranges, one per CTA, so every SM streams the same number of
//               bytes whatever N and K are;
//   stage     = up to 4 column blocks of one band, 5 copies: the codes (one contiguous
//               bulk copy), the activations (one 3-D TMA box of 4 column blocks x 8*NT
//               token rows, 128B swizzle, rows >= M zero-filled), the s_inv slice, and the
//               group rows of scales and of zero points met by the stage (2-D TMA boxes);
//   CTA       = 1 producer warp + 8 consumer warps; consumer warp w owns rows
//               16w..16w+15 of the band; per 16-deep step one 32-bit word per lane is
//               unpacked into the A operand of mma.m16n8k16 (weights as the 16-row side,
//               up to 64 tokens as 8-column tiles), multiplied as exact integers (q - z)
//               with fp32 accumulation; each group's partial sum is scaled in fp32;
//   fix-up    = a band split between CTAs is completed by the last CTA to finish it,
//               which adds the fp32 partials of all contributors in CTA order
//               (deterministic) and stores Y; its counter is reset to zero.
#pragma once
#include "w4_common.cuh"

namespace w4d {

constexpr int kWarps = 8;                 // consumer warps = row tiles per band
constexpr int kBandRows = 16 * kWarps;    // 128
constexpr int kAtomsPerStage = 4;         // column blocks per stage (256 input channels)
constexpr int kThreads = 32 * (kWarps + 1);

template <int NT>
struct Cfg {
    static constexpr int stages = NT == 1 ? 4 : 3;
    static constexpr int mpad = 8 * NT;               // token rows per activation box slot
    static constexpr int xbox = mpad * 128;           // bytes per activation box slot
};

struct DecodeParams {
    const uint32_t* qw;       // device layout
    const __half* scales;     // [G,N]
    const __half* zeros;      // [G,N] or null
    const int32_t* g_idx;     // [K] or null
    const float* s_inv;       // [K] or null
    void* Y;                  // [M,N]
    float* partials;          // [P][2][128][8*NT] fp32 (workspace)
    unsigned* counters;       // [bands] (workspace, zero between calls)
    int M, N, K, group_size, G, out_dtype;
    int KA;                   // K / 64
    int tiles;                // N / 16
    int units;                // bands * KA atoms
    int base, rem;            // atoms per CTA: base (+1 for the first rem CTAs)
    int ngs;                  // group rows staged per stage (scale / zero-point box height)
    // byte offsets inside one stage
    int off_x, off_si, off_sc, off_zr, off_gi, stage_bytes;
};

W4_DEV int unit_begin(const DecodeParams& p, int c) { return c * p.base + min(c, p.rem); }
W4_DEV int cta_of_unit(const DecodeParams& p, int u) {
    const int split = p.rem * (p.base + 1);
    return u < split ? u / (p.base + 1) : p.rem + (u - split) / p.base;
}
W4_DEV int band_tiles(const DecodeParams& p, int band) { return min(kWarps, p.tiles - band * kWarps); }

W4_DEV void store_out(const DecodeParams& p, int m, int n, float v) {
    const size_t idx = (size_t)m * p.N + n;
    if (p.out_dtype == 2) reinterpret_cast<float*>(p.Y)[idx] = v;
    else if (p.out_dtype == 1) reinterpret_cast<__nv_bfloat16*>(p.Y)[idx] = __float2bfloat16_rn(v);
    else reinterpret_cast<__half*>(p.Y)[idx] = __float2half_rn(v);
}

W4_DEV uint32_t lds32(const unsigned char* p) { return *reinterpret_cast<const uint32_t*>(p); }
W4_DEV uint32_t lds32_at(uint32_t saddr) {
    uint32_t v;
    asm volatile("ld.shared.b32 %0, [%1];" : "=r"(v) : "r"(saddr));
    return v;
}

// byte offset of the 4-byte pair (token row, k-pair kp < 32) inside a 128B-swizzled box
W4_DEV int xsw(int tok, int kp) { return tok * 128 + (((kp >> 2) ^ (tok & 7)) << 4) + ((kp & 3) << 2); }

// Complete or hand off the accumulators of one band.
template <int NT>
W4_DEV void flush_band(const DecodeParams& p, int band, int u0, int u1, int cta, int w,
                       int lane, int ctid, bool aborted, float (&acc)[NT][4],
                       volatile int* s_flag) {
    const int Mp = 8 * NT;
    const bool tile_ok = w < band_tiles(p, band);
    const int rl0 = 16 * w + (lane >> 2);            // row within the band
    const int n0 = band * kBandRows + rl0;
    const int q2 = 2 * (lane & 3);
    const bool whole = (u0 <= band * p.KA) && (u1 >= (band + 1) * p.KA);
    if (whole) {
        if (tile_ok && !aborted) {
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = 8 * nt + q2 + (e & 1);
                    const int n = n0 + ((e >> 1) << 3);
                    if (m < p.M) store_out(p, m, n, acc[nt][e]);
                }
        }
        return;
    }
    // partial band: write this CTA's fp32 partial sums to its slot
    const int first_band = unit_begin(p, cta) / p.KA;
    const int which = (band == first_band) ? 0 : 1;
    float* slot = p.partials + ((size_t)cta * 2 + which) * (size_t)(kBandRows * Mp);
    if (tile_ok && !aborted) {
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = 8 * nt + q2 + (e & 1);
                const int rl = rl0 + ((e >> 1) << 3);
                if (m < p.M) slot[rl * Mp + m] = acc[nt][e];
            }
    }
    __threadfence();
    named_bar_sync(2, 32 * kWarps);
    const int c_first = cta_of_unit(p, band * p.KA);
    const int c_last = cta_of_unit(p, (band + 1) * p.KA - 1);
    if (ctid == 0) {
        int last = 0;
        if (!aborted) {
            const unsigned prev = atomicAdd(p.counters + band, 1u);
            last = (prev == (unsigned)(c_last - c_first));
        }
        *s_flag = last;
    }
    named_bar_sync(2, 32 * kWarps);
    if (*s_flag) {
        __threadfence();
        if (tile_ok) {
            // Only the first contributor can hold this band in its second slot (its range
            // began in an earlier band); every later one began inside this band.
            const int first_slot = (unit_begin(p, c_first) < band * p.KA) ? 1 : 0;
            const size_t slot_elems = (size_t)kBandRows * Mp;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = 8 * nt + q2 + (e & 1);
                    const int rl = rl0 + ((e >> 1) << 3);
                    if (m >= p.M) continue;
                    const float* base = p.partials + rl * Mp + m;
                    float v = 0.0f;
                    // contributors in CTA order, loads issued a batch at a time
                    for (int cb = c_first; cb <= c_last; cb += 8) {
                        float part[8];
#pragma unroll
                        for (int t = 0; t < 8; ++t) {
                            const int c = cb + t;
                            const int wc = (c == c_first) ? first_slot : 0;
                            part[t] = (c <= c_last) ? __ldcg(base + ((size_t)c * 2 + wc) * slot_elems) : 0.0f;
                        }
#pragma unroll
                        for (int t = 0; t < 8; ++t) v += part[t];
                    }
                    store_out(p, m, band * kBandRows + rl, v);
                }
        }
        if (ctid == 0) p.counters[band] = 0u;
    }
    named_bar_sync(2, 32 * kWarps);
}

W4_DEV void fold(float s0, float s1, float (&c)[4], float (&acc)[4]) {
    acc[0] = fmaf(s0, c[0], acc[0]);
    acc[1] = fmaf(s0, c[1], acc[1]);
    acc[2] = fmaf(s1, c[2], acc[2]);
    acc[3] = fmaf(s1, c[3], acc[3]);
    c[0] = c[1] = c[2] = c[3] = 0.0f;
}

// One stage of the decode consumer (contiguous groups): the warp's 16-row tile times
// up to kAtomsPerStage column blocks staged at `st`; partial sums of each group are
// folded into acc with the group's fp32 scale.  nb = first column of the next group.
template <int NT, bool BF16>
W4_DEV void consume_stage(const unsigned char* st, int off_x, int off_sc, int off_zr, bool has_zeros,
                          int na, int a0, int tb, int nb, int g, bool g32, int w, int lane,
                          int rl0, int rl1, uint32_t xrow, const int (&xlo)[4], const int (&xhi)[4],
                          const ZeroConsts& zc_sym, float (&acc)[NT][4]) {
    using C = Cfg<NT>;
    const __half* scp = reinterpret_cast<const __half*>(st + off_sc);
    const unsigned short* zrp = reinterpret_cast<const unsigned short*>(st + off_zr);
    float s0 = __half2float(scp[rl0]), s1 = __half2float(scp[rl1]);
    ZeroConsts zc = has_zeros ? zero_consts_h<BF16>(zrp[rl0], zrp[rl1]) : zc_sym;
    // two accumulator chains (even / odd 16-deep steps) for MMA overlap
    float c0[NT][4], c1[NT][4];
#pragma unroll
    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
        for (int e = 0; e < 4; ++e) c0[nt][e] = c1[nt][e] = 0.0f;
    // per-stage fragment base addresses: every load below is one of these registers plus
    // a compile-time offset
    uint32_t xl[4], xh[4];
    const uint32_t xs = smem_u32(st + off_x) + xrow;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        xl[j] = xs + xlo[j];
        xh[j] = xs + xhi[j];
    }
    const unsigned char* wbase = st + w * 512 + lane * 16;
    const int wstride = tb * 512;
    int ka = 64 * a0;
#pragma unroll
    for (int a = 0; a < kAtomsPerStage; ++a) {
        if (a < na) {
            const uint4 wq = *reinterpret_cast<const uint4*>(wbase + a * wstride);
            const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                if ((j == 0 || (j == 2 && g32)) && ka + 16 * j >= nb) {
                    // group boundary: fold the finished group's partials, load the next
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        fold(s0, s1, c0[nt], acc[nt]);
                        fold(s0, s1, c1[nt], acc[nt]);
                    }
                    nb += g;
                    scp += 128;
                    zrp += 128;
                    s0 = __half2float(scp[rl0]);
                    s1 = __half2float(scp[rl1]);
                    if (has_zeros) zc = zero_consts_h<BF16>(zrp[rl0], zrp[rl1]);
                }
                uint32_t af[4];
                unpack_word<BF16>(wv[j], zc, af);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    // token rows >= M were zero-filled by the tensor copy
                    const uint32_t b0 = lds32_at(xl[j] + a * C::xbox + nt * 1024);
                    const uint32_t b1 = lds32_at(xh[j] + a * C::xbox + nt * 1024);
                    // with few token tiles a second chain breaks the MMA dependency; with
                    // more tiles they already interleave
                    mma_16816<BF16>((NT <= 2 && (j & 1)) ? c1[nt] : c0[nt], af, b0, b1);
                }
            }
            ka += 64;
        }
    }
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) {
        fold(s0, s1, c0[nt], acc[nt]);
        fold(s0, s1, c1[nt], acc[nt]);
    }
}

template <int NT, bool BF16, bool GIDX>
__global__ void __launch_bounds__(kThreads, NT >= 8 ? 1 : 2)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_sc,
                  const __grid_constant__ CUtensorMap tmap_zr, const DecodeParams p) {
    using C = Cfg<NT>;
    constexpr int S = C::stages;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = reinterpret_cast<unsigned char*>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + S * p.stage_bytes);
    uint64_t* empty = full + S;
    volatile int* s_abort = reinterpret_cast<volatile int*>(empty + S);
    volatile int* s_last = s_abort + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const int u0 = unit_begin(p, cta), u1 = unit_begin(p, cta + 1);
    const int g = p.group_size;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWarps);
        }
        *s_abort = 0;
        *s_last = 0;
        fence_mbar_init();
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tmap_x);
        if (!GIDX) {
            prefetch_tensormap(&tmap_sc);
            if (p.zeros) prefetch_tensormap(&tmap_zr);
        }
    }
    __syncthreads();
    // The next kernel may be scheduled as soon as every CTA of this grid is running.
    // Everything this kernel reads before pdl_wait() (codes, scales, zero points, g_idx)
    // is never written by the kernels of this library.
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t policy = policy_evict_first();
        int i = 0;
        for (int u = u0; u < u1; ++i) {
            const int band = u / p.KA, a0 = u - band * p.KA;
            const int na = min(kAtomsPerStage, min(p.KA - a0, u1 - u));
            const int s = i % S, ph = (i / S) & 1;
            if (i >= S) {
                const bool ok = !*s_abort && mbar_wait(&empty[s], ph ^ 1);
                if (!ok) { *s_abort = 1; break; }
            }
            unsigned char* st = smem + s * p.stage_bytes;
            const int tb = band_tiles(p, band);
            // one copy per operand: codes (contiguous run of the band), activations (one
            // 3-D box: 4 column blocks x 8*NT token rows, rows >= M and blocks beyond K
            // zero-filled), s_inv slice, scale rows and zero-point rows (2-D boxes).  The
            // read-only weight operands of the first stages go out before pdl_wait(), the
            // activations (possibly produced by the preceding kernel) after it.
            const int g_first = (64 * a0) / g;
            uint32_t bytes = na * tb * 512 + kAtomsPerStage * C::xbox;
            if (p.s_inv) bytes += na * 256;
            if (GIDX) bytes += na * 256;
            else bytes += p.ngs * 256 * (p.zeros ? 2 : 1);
            if (lane == 0) {
                mbar_arrive_expect_tx(&full[s], bytes);
                bulk_g2s_hint(st, p.qw + 128 * ((size_t)8 * p.KA * band + (size_t)a0 * tb),
                              na * tb * 512, &full[s], policy);
                if (GIDX) {
                    bulk_g2s(st + p.off_gi, p.g_idx + 64 * a0, na * 256, &full[s]);
                } else {
                    tma_load_2d(st + p.off_sc, &tmap_sc, band * kBandRows, g_first, &full[s]);
                    if (p.zeros) tma_load_2d(st + p.off_zr, &tmap_zr, band * kBandRows, g_first, &full[s]);
                }
                if (i == 0) pdl_wait();
                tma_load_3d(st + p.off_x, &tmap_x, 0, 0, a0, &full[s]);
                if (p.s_inv) bulk_g2s(st + p.off_si, p.s_inv + 64 * a0, na * 256, &full[s]);
            }
            __syncwarp();
            u += na;
        }
        // On abort, wait (bounded) for the copies already issued before leaving.
        if (*s_abort && lane == 0)
            for (int k = (i > S ? i - S : 0); k < i; ++k) (void)mbar_wait(&full[k % S], (k / S) & 1);
    } else {
        // ------------------------------------------------------------ consumers
        pdl_wait();   // before any store to Y or the workspace
        const int w = warp - 1;
        const int ctid = threadIdx.x - 32;
        const int q = lane & 3, g8 = lane >> 2;
        const int rl0 = 16 * w + g8, rl1 = rl0 + 8;
        // activation fragment offsets inside a 128B-swizzled box: row g8 (+8 per token
        // tile), k pairs 8j+q (b0) and 8j+4+q (b1) of the 16-deep step j
        const uint32_t xrow = g8 * 128;
        int xlo[4], xhi[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xlo[j] = (((2 * j) ^ g8) << 4) + 4 * q;
            xhi[j] = (((2 * j + 1) ^ g8) << 4) + 4 * q;
        }
        const bool g32 = (g == 32);
        // symmetric format: the implicit zero point 8 never changes
        const ZeroConsts zc_sym = zero_consts_h<BF16>(0x4800u, 0x4800u);
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
        // stage coordinates advance incrementally (one division per CTA)
        int band = (u0 < u1) ? u0 / p.KA : 0;
        int a0 = u0 - band * p.KA;
        int cur_band = (u0 < u1) ? band : -1;
        int gcur = (64 * a0) / g;          // group of the next column to process
        int next_b = (gcur + 1) * g;       // first column of the following group
        bool aborted = false;

        int i = 0;
        for (int u = u0; u < u1; ++i) {
            const int na = min(kAtomsPerStage, min(p.KA - a0, u1 - u));
            const int s = i % S, ph = (i / S) & 1;
            if (band != cur_band) {
                flush_band<NT>(p, cur_band, u0, u1, cta, w, lane, ctid, aborted, acc, s_last);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
                cur_band = band;
            }
            if (!aborted) {
                aborted = *s_abort || !mbar_wait(&full[s], ph);
                if (aborted) *s_abort = 1;
            }
            unsigned char* st = smem + s * p.stage_bytes;
            unsigned char* xb = st + p.off_x;
            if (p.s_inv) {
                // X' = X * s_inv rounded to the activation type, in place, once per stage
                if (!aborted) {
                    const float* si = reinterpret_cast<const float*>(st + p.off_si);
                    const int per_box = p.M * 32;
#pragma unroll
                    for (int a = 0; a < kAtomsPerStage; ++a) {
                        if (a < na) {
                            for (int r = ctid; r < per_box; r += 32 * kWarps) {
                                const int tok = r >> 5, kp = r & 31;
                                uint32_t* px = reinterpret_cast<uint32_t*>(xb + a * C::xbox + xsw(tok, kp));
                                const float2 v = unpack2<BF16>(*px);
                                const float2 sv = *reinterpret_cast<const float2*>(si + 64 * a + 2 * kp);
                                *px = pack2<BF16>(__fmul_rn(v.x, sv.x), __fmul_rn(v.y, sv.y));
                            }
                        }
                    }
                }
                named_bar_sync(1, 32 * kWarps);
            }
            const int tb = band_tiles(p, band);
            if (!GIDX) {
                // the group containing this stage's first column (the staged scale and
                // zero-point rows start there)
                while (64 * a0 >= next_b) {
                    next_b += g;
                    ++gcur;
                }
            }
            if (!aborted && w < tb) {
                if constexpr (!GIDX) {
                    consume_stage<NT, BF16>(st, p.off_x, p.off_sc, p.off_zr, p.zeros != nullptr, na, a0,
                                            tb, next_b, g, g32, w, lane, rl0, rl1, xrow, xlo, xhi,
                                            zc_sym, acc);
                } else {
                    // act-order: every channel has its own group; fold the scale into an
                    // fp16 weight (q - z) * scale before the MMA
                    const int32_t* gis = reinterpret_cast<const int32_t*>(st + p.off_gi);
                    const int n_r0 = band * kBandRows + rl0, n_r1 = n_r0 + 8;
#pragma unroll
                    for (int a = 0; a < kAtomsPerStage; ++a) {
                        if (a < na) {
                            const uint4 wq = *reinterpret_cast<const uint4*>(
                                st + (a * tb + w) * 512 + lane * 16);
                            const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
                            const unsigned char* xa = xb + a * C::xbox;
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const int kk = 64 * a + 16 * j + 2 * q;
                                int gk[4] = {gis[kk], gis[kk + 1], gis[kk + 8], gis[kk + 9]};
#pragma unroll
                                for (int e = 0; e < 4; ++e)
                                    if (gk[e] < 0 || gk[e] >= p.G) {
                                        atomicOr(&g_w4_error_word, W4_DEVERR_GIDX);
                                        gk[e] = 0;
                                    }
                                uint32_t af[4];
#pragma unroll
                                for (int r = 0; r < 4; ++r) {
                                    const int row = (r & 1) ? n_r1 : n_r0;
                                    const int kl = (r & 2) ? 2 : 0;
                                    const float qlo = (float)((wv[j] >> (4 * r)) & 0xF);
                                    const float qhi = (float)((wv[j] >> (4 * (r + 4))) & 0xF);
                                    const __half z_lo = p.zeros ? __ldg(p.zeros + (size_t)gk[kl] * p.N + row)
                                                                : __float2half_rn(8.0f);
                                    const __half z_hi = p.zeros ? __ldg(p.zeros + (size_t)gk[kl + 1] * p.N + row)
                                                                : __float2half_rn(8.0f);
                                    const __half2 ss = __halves2half2(__ldg(p.scales + (size_t)gk[kl] * p.N + row),
                                                                      __ldg(p.scales + (size_t)gk[kl + 1] * p.N + row));
                                    af[r] = h2_as_u32(__hmul2(
                                        __hsub2(__floats2half2_rn(qlo, qhi), __halves2half2(z_lo, z_hi)), ss));
                                }
#pragma unroll
                                for (int nt = 0; nt < NT; ++nt) {
                                    const uint32_t b0 = lds32(xa + xrow + nt * 1024 + xlo[j]);
                                    const uint32_t b1 = lds32(xa + xrow + nt * 1024 + xhi[j]);
                                    mma_16816<false>(acc[nt], af, b0, b1);
                                }
                            }
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
            u += na;
            a0 += na;
            if (a0 == p.KA) {
                a0 = 0;
                ++band;
                gcur = 0;
                next_b = g;
            }
        }
        if (cur_band >= 0)
            flush_band<NT>(p, cur_band, u0, u1, cta, w, lane, ctid, aborted, acc, s_last);
    }
}

}  // namespace w4d
