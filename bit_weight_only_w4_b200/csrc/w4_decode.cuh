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
//   unit      = 128 output rows (8 tiles of 16) x 64 input channels; the units of the
//               layer are ordered row-band-major and split into equal contiguous
//               ranges, one per CTA (stream-K), so every SM streams the same number of
//               bytes whatever N and K are;
//   CTA       = 1 producer warp (one elected lane drives TMA bulk copies into an
//               8-stage shared-memory ring) + 8 consumer warps (warp w owns rows
//               16w..16w+15 of the band);
//   consumer  = for each 16-deep step, one 32-bit word per lane is unpacked into the
//               A operand of mma.m16n8k16 (weights as the 16-row side, up to 64 tokens
//               as 8-column tiles), multiplied by exact integer weights (q - z) with
//               fp32 accumulation, and each group's partial sum is multiplied by its
//               scale in fp32;
//   fix-up    = a band split between CTAs is completed by the last CTA to finish it,
//               which adds the fp32 partials of all contributors in CTA order
//               (deterministic) and stores Y; its counter is reset to zero.
#pragma once
#include "w4_common.cuh"

namespace w4d {

constexpr int kWarps = 8;                 // consumer warps = row tiles per band
constexpr int kBandRows = 16 * kWarps;    // 128
constexpr int kStages = 8;
constexpr int kXRow = 144;                // bytes per token row of a staged activation chunk
constexpr int kThreads = 32 * (kWarps + 1);

// shared-memory layout of one ring stage
template <int NT>
struct StageLayout {
    static constexpr int w = 0;                         // 8 tiles x 512 B packed weights
    static constexpr int x = 4096;                      // up to 8*NT rows x 144 B
    static constexpr int si = x + 8 * NT * kXRow;       // 64 fp32 s_inv
    static constexpr int sc = si + 256;                 // up to 2 groups x 128 fp16 scales
    static constexpr int zr = sc + 512;                 // up to 2 groups x 128 fp16 zeros
    static constexpr int gi = zr + 512;                 // 64 int32 g_idx
    static constexpr int bytes = ((gi + 256) + 127) / 128 * 128;
};

template <int NT>
struct SmemLayout {
    static constexpr int ring = 0;
    static constexpr int xc = ring + kStages * StageLayout<NT>::bytes;   // 2 converted chunks
    static constexpr int bars = xc + 2 * 8 * NT * kXRow;
    static constexpr int flags = bars + 2 * kStages * 8;
    static constexpr int bytes = flags + 16;
};

struct DecodeParams {
    const void* X;            // [M,K] fp16/bf16
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
    int units;                // bands * KA
    int base, rem;            // units per CTA: base (+1 for the first rem CTAs)
};

W4_DEV int unit_begin(const DecodeParams& p, int c) { return c * p.base + min(c, p.rem); }
W4_DEV int cta_of_unit(const DecodeParams& p, int u) {
    const int split = p.rem * (p.base + 1);
    return u < split ? u / (p.base + 1) : p.rem + (u - split) / p.base;
}

W4_DEV void store_out(const DecodeParams& p, int m, int n, float v) {
    const size_t idx = (size_t)m * p.N + n;
    if (p.out_dtype == 2) reinterpret_cast<float*>(p.Y)[idx] = v;
    else if (p.out_dtype == 1) reinterpret_cast<__nv_bfloat16*>(p.Y)[idx] = __float2bfloat16_rn(v);
    else reinterpret_cast<__half*>(p.Y)[idx] = __float2half_rn(v);
}

W4_DEV uint32_t lds32(const unsigned char* p) { return *reinterpret_cast<const uint32_t*>(p); }

// Complete or hand off the accumulators of one band.
template <int NT>
W4_DEV void flush_band(const DecodeParams& p, int band, int u0, int u1, int cta, int w,
                       int lane, int ctid, bool tile_ok, bool aborted,
                       float (&acc)[NT][4], volatile int* s_flag) {
    const int Mp = 8 * NT;
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
                slot[rl * Mp + m] = acc[nt][e];
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
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int m = 8 * nt + q2 + (e & 1);
                    const int rl = rl0 + ((e >> 1) << 3);
                    if (m >= p.M) continue;
                    float v = 0.0f;
                    for (int c = c_first; c <= c_last; ++c) {
                        const int wc = (unit_begin(p, c) / p.KA == band) ? 0 : 1;
                        v += __ldcg(p.partials + ((size_t)c * 2 + wc) * (size_t)(kBandRows * Mp) +
                                    rl * Mp + m);
                    }
                    store_out(p, m, band * kBandRows + rl, v);
                }
        }
        if (ctid == 0) p.counters[band] = 0u;
    }
    named_bar_sync(2, 32 * kWarps);
}

template <int NT, bool BF16, bool GIDX>
__global__ void __launch_bounds__(kThreads, NT >= 8 ? 1 : 2) decode_kernel(const DecodeParams p) {
    using SL = StageLayout<NT>;
    using ML = SmemLayout<NT>;
    extern __shared__ __align__(128) unsigned char smem[];
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + ML::bars);
    uint64_t* empty = full + kStages;
    volatile int* s_abort = reinterpret_cast<volatile int*>(smem + ML::flags);
    volatile int* s_last = s_abort + 1;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const int u0 = unit_begin(p, cta), u1 = unit_begin(p, cta + 1);
    const int ngroups = (p.group_size == 32) ? 2 : 1;   // groups met by one 64-deep unit

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], kWarps);
        }
        *s_abort = 0;
        *s_last = 0;
        fence_mbar_init();
    }
    __syncthreads();

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        const uint64_t policy = policy_evict_first();
        int issued = 0;
        for (int u = u0; u < u1; ++u, ++issued) {
            const int i = u - u0, s = i % kStages, ph = (i / kStages) & 1;
            if (i >= kStages) {
                bool ok = !*s_abort && mbar_wait(&empty[s], ph ^ 1);
                if (!ok) { *s_abort = 1; break; }
            }
            unsigned char* st = smem + s * SL::bytes;
            const int band = u / p.KA, a = u - band * p.KA;
            const int tiles = min(kWarps, p.tiles - band * kWarps);
            const int rows = 16 * tiles;
            uint32_t bytes = tiles * 512 + p.M * 128;
            if (p.s_inv) bytes += 256;
            if (GIDX) bytes += 256;
            else bytes += ngroups * rows * 2 * (p.zeros ? 2 : 1);
            if (lane == 0) mbar_arrive_expect_tx(&full[s], bytes);
            __syncwarp();
            for (int c = lane; c < tiles; c += 32)
                bulk_g2s_hint(st + SL::w + c * 512,
                              p.qw + ((size_t)(band * kWarps + c) * p.KA + a) * 128, 512,
                              &full[s], policy);
            for (int c = lane; c < p.M; c += 32)
                bulk_g2s(st + SL::x + c * kXRow,
                         reinterpret_cast<const unsigned char*>(p.X) +
                             ((size_t)c * p.K + (size_t)a * 64) * 2,
                         128, &full[s]);
            if (lane == 0 && p.s_inv) bulk_g2s(st + SL::si, p.s_inv + a * 64, 256, &full[s]);
            if (GIDX) {
                if (lane == 1) bulk_g2s(st + SL::gi, p.g_idx + a * 64, 256, &full[s]);
            } else if (lane >= 2 && lane < 2 + ngroups) {
                const int gg = lane - 2;
                const int grp = (a * 64) / p.group_size + gg;
                const size_t off = (size_t)grp * p.N + (size_t)band * kBandRows;
                bulk_g2s(st + SL::sc + gg * 256, p.scales + off, rows * 2, &full[s]);
                if (p.zeros) bulk_g2s(st + SL::zr + gg * 256, p.zeros + off, rows * 2, &full[s]);
            }
            __syncwarp();
        }
        // On abort, wait (bounded) for copies already issued before leaving.
        if (*s_abort && lane == 0) {
            for (int i = (issued > kStages ? issued - kStages : 0); i < issued; ++i)
                (void)mbar_wait(&full[i % kStages], (i / kStages) & 1);
        }
    } else {
        // ------------------------------------------------------------ consumers
        const int w = warp - 1;
        const int ctid = threadIdx.x - 32;
        const int q = lane & 3, g8 = lane >> 2;
        const int rl0 = 16 * w + g8, rl1 = rl0 + 8;
        float acc[NT][4];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[nt][e] = 0.0f;
        int cur_band = (u0 < u1) ? u0 / p.KA : -1;
        bool aborted = false;

        for (int u = u0; u < u1; ++u) {
            const int i = u - u0, s = i % kStages, ph = (i / kStages) & 1;
            const int band = u / p.KA;
            const bool tile_ok = band * kWarps + w < p.tiles;
            if (band != cur_band) {
                flush_band<NT>(p, cur_band, u0, u1, cta, w, lane, ctid,
                               cur_band * kWarps + w < p.tiles, aborted, acc, s_last);
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
            const unsigned char* st = smem + s * SL::bytes;
            const unsigned char* xb = st + SL::x;
            if (p.s_inv) {
                // X' = X * s_inv, rounded to the activation type, once per chunk for all warps
                unsigned char* xc = smem + ML::xc + (i & 1) * (8 * NT * kXRow);
                if (!aborted) {
                    for (int e = ctid; e < p.M * 32; e += 32 * kWarps) {
                        const int tok = e >> 5, kp = e & 31;
                        const float2 v = unpack2<BF16>(lds32(xb + tok * kXRow + kp * 4));
                        const float2 si = *reinterpret_cast<const float2*>(st + SL::si + kp * 8);
                        *reinterpret_cast<uint32_t*>(xc + tok * kXRow + kp * 4) =
                            pack2<BF16>(__fmul_rn(v.x, si.x), __fmul_rn(v.y, si.y));
                    }
                }
                named_bar_sync(1, 32 * kWarps);
                xb = xc;
            }
            if (!aborted && tile_ok) {
                const uint4 wq = *reinterpret_cast<const uint4*>(st + SL::w + w * 512 + lane * 16);
                const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
                if constexpr (!GIDX) {
                    // scale and zero-point constants of the (at most two) groups of this unit
                    const bool two = (ngroups == 2);
                    const __half* sca = reinterpret_cast<const __half*>(st + SL::sc);
                    const __half* zra = reinterpret_cast<const __half*>(st + SL::zr);
                    const float sa0 = __half2float(sca[rl0]), sa1 = __half2float(sca[rl1]);
                    const float sb0 = two ? __half2float(sca[128 + rl0]) : sa0;
                    const float sb1 = two ? __half2float(sca[128 + rl1]) : sa1;
                    float za0 = 8.0f, za1 = 8.0f, zb0 = 8.0f, zb1 = 8.0f;
                    if (p.zeros) {
                        za0 = __half2float(zra[rl0]);
                        za1 = __half2float(zra[rl1]);
                        zb0 = two ? __half2float(zra[128 + rl0]) : za0;
                        zb1 = two ? __half2float(zra[128 + rl1]) : za1;
                    }
                    const ZeroConsts zca = BF16 ? zero_consts_bf16(za0, za1) : zero_consts_f16(za0, za1);
                    const ZeroConsts zcb = BF16 ? zero_consts_bf16(zb0, zb1) : zero_consts_f16(zb0, zb1);
                    float c[NT][4];
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) c[nt][e] = 0.0f;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        uint32_t af[4];
                        unpack_word<BF16>(wv[j], j < 2 ? zca : zcb, af);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const int tok = 8 * nt + g8;
                            uint32_t b0 = 0, b1 = 0;
                            if (tok < p.M) {
                                const unsigned char* xr = xb + tok * kXRow + (16 * j + 2 * q) * 2;
                                b0 = lds32(xr);
                                b1 = lds32(xr + 16);
                            }
                            mma_16816<BF16>(c[nt], af, b0, b1);
                        }
                        // end of a group: fold the group's partial into the accumulators
                        if (j == 3 || (j == 1 && two)) {
                            const float s0 = j < 2 ? sa0 : sb0;
                            const float s1 = j < 2 ? sa1 : sb1;
#pragma unroll
                            for (int nt = 0; nt < NT; ++nt) {
                                acc[nt][0] = fmaf(s0, c[nt][0], acc[nt][0]);
                                acc[nt][1] = fmaf(s0, c[nt][1], acc[nt][1]);
                                acc[nt][2] = fmaf(s1, c[nt][2], acc[nt][2]);
                                acc[nt][3] = fmaf(s1, c[nt][3], acc[nt][3]);
                                c[nt][0] = c[nt][1] = c[nt][2] = c[nt][3] = 0.0f;
                            }
                        }
                    }
                } else {
                    // act-order: every channel has its own group; fold the scale into an
                    // fp16 weight (q - z) * scale before the MMA
                    const int32_t* gis = reinterpret_cast<const int32_t*>(st + SL::gi);
                    const int n_r0 = band * kBandRows + rl0, n_r1 = n_r0 + 8;
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int kk = 16 * j + 2 * q;
                        int gk[4] = {gis[kk], gis[kk + 1], gis[kk + 8], gis[kk + 9]};
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (gk[e] < 0 || gk[e] >= p.G) {
                                atomicOr(&g_w4_error_word, W4_DEVERR_GIDX);
                                gk[e] = 0;
                            }
                        auto sc_of = [&](int g, int n) {
                            return __ldg(p.scales + (size_t)g * p.N + n);
                        };
                        auto z_of = [&](int g, int n) {
                            return p.zeros ? __ldg(p.zeros + (size_t)g * p.N + n) : __float2half_rn(8.0f);
                        };
                        const uint32_t wj = wv[j];
                        // codes in the order of the A registers: (r0: c,c+1) (r1: c,c+1)
                        // (r0: c+8,c+9) (r1: c+8,c+9) = nibbles (0,4) (1,5) (2,6) (3,7)
                        uint32_t af[4];
#pragma unroll
                        for (int r = 0; r < 4; ++r) {
                            const int row = (r & 1) ? n_r1 : n_r0;
                            const int klo = (r & 2) ? 2 : 0;   // index into gk
                            const float qlo = (float)((wj >> (4 * r)) & 0xF);
                            const float qhi = (float)((wj >> (4 * (r + 4))) & 0xF);
                            const __half2 qq = __floats2half2_rn(qlo, qhi);
                            const __half2 zz = __halves2half2(z_of(gk[klo], row), z_of(gk[klo + 1], row));
                            const __half2 ss = __halves2half2(sc_of(gk[klo], row), sc_of(gk[klo + 1], row));
                            af[r] = h2_as_u32(__hmul2(__hsub2(qq, zz), ss));
                        }
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            const int tok = 8 * nt + g8;
                            uint32_t b0 = 0, b1 = 0;
                            if (tok < p.M) {
                                const unsigned char* xr = xb + tok * kXRow + (16 * j + 2 * q) * 2;
                                b0 = lds32(xr);
                                b1 = lds32(xr + 16);
                            }
                            mma_16816<false>(acc[nt], af, b0, b1);
                        }
                    }
                }
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&empty[s]);
        }
        if (cur_band >= 0)
            flush_band<NT>(p, cur_band, u0, u1, cta, w, lane, ctid,
                           cur_band * kWarps + w < p.tiles, aborted, acc, s_last);
    }
}

}  // namespace w4d
