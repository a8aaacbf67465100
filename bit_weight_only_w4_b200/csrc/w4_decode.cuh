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
//               128-row band are stored column block by column block, so consecutive
//               column blocks of a band are one contiguous copy;
//   unit      = 2 column blocks (128 input channels) of one band; all units of the layer
//               are split into equal contiguous ranges, one per CTA (stream-K), so every
//               SM streams the same number of bytes whatever N and K are;
//   stage     = up to 4 units of one band (32 KB of codes, one bulk copy) and the group
//               rows of scales and zero points (2-D boxes); staged activations add a 3-D
//               TMA box of the stage's column blocks x 8*NT token rows of the prepared X'
//               (rows >= M zero-filled) and three bulk copies of its sums;
//   CTA       = 1 producer warp (lane 0 issues a stage's copies) and 16 MMA warps in two
//               groups that take alternate stages (8 in one group with 4 or 8 token
//               tiles); one CTA per SM, its ring filling the SM's shared memory, so every
//               SM holds exactly one CTA of a GEMM even when the next GEMM's CTAs start
//               early under programmatic dependent launch;
//   activations= with one token tile and a small M*K, X' = X * s_inv and its sums over 32,
//               64 and 128 channels are prepared by every CTA for the input channels of
//               its own units and stay resident (with act-order weights packed in
//               permuted order, gathered through perm); otherwise prep_acts_kernel
//               prepares them once per GEMM in the workspace, and each stage copies its
//               slice;
//   zero point= the MMA multiplies the biased codes o + m*q (o + m*q is what the AND/OR
//               unpack yields; no subtraction per weight) and the per-group fold removes
//               the bias and the zero point with the activation sums S = sum_k X'[m,k] of
//               the group: sum_k (q-z) X' = (c - (o + m*z) S) / m, in fp32;
//   fix-up    = a band split between CTAs is completed by the CTA holding its last unit;
//               a CTA processes its contributor part first (publishing fp32 partials as
//               {value, flag} words), its whole bands next and the completing part last,
//               after which all MMA threads sum the contributors' shares in CTA order
//               (deterministic, no atomics).
#pragma once
#include "w4_common.cuh"
#include "w4_fp4.cuh"

namespace w4d {

constexpr int kBandRows = 128;
constexpr int kTilesPerBand = 8;

// Group handling of the MMA warps.
enum : int {
    kModeHalf = 0,   // group size a multiple of 128, K a multiple of 128: one fold per half stage
    kModeAtom = 1,   // group size a multiple of 64: folds at 64-channel boundaries
    kModeG32 = 2,    // group size 32: folds every 32 channels
    kModeGidx = 3,   // act-order g_idx: the scale is folded into each fp16 weight
    kModeNvfp4 = 4,  // NVFP4 weights: E2M1 decoded to fp16, E4M3 block scale per 16 channels
    kModeMxfp4 = 5,  // MXFP4 weights: E2M1 decoded to fp16, power-of-two scale per 32 channels
};

template <int NT>
struct Cfg {
    static constexpr int tpw = NT <= 2 ? 2 : 1;          // row tiles per MMA warp
    static constexpr int aps = 8;                        // atoms (64-channel blocks) per stage: 32 KB of codes
    // no activation warps: X' and its sums arrive prepared (resident, or copied per stage
    // from the copy prep_acts_kernel wrote); every warp but the producer is an MMA warp
    static constexpr int xw = 0;
    // 17 warps with one or two token tiles; 9 with more, so that their larger
    // accumulator sets fit the registers (9 warps allow 168 a thread)
    static constexpr int mma_warps = NT <= 2 ? 16 : 8;
    static constexpr int groups = mma_warps / 8;         // stage-parity groups
    static constexpr int stage_warps = mma_warps / groups;   // MMA warps sharing a stage
    static constexpr int tsets = 8 / tpw;                // row-tile sets of a band
    static constexpr int kparts = stage_warps / tsets;   // K slices of a stage
    static constexpr int apk = aps / kparts;             // atoms per K slice
    static constexpr int warps = 1 + xw + mma_warps;
    static constexpr int threads = 32 * warps;
    static constexpr int mpad = 8 * NT;                  // token rows per activation box slot
    // activation sums of one stage: per token, over 32, 64 and 128 consecutive channels
    static constexpr int sx32 = 0, sx64 = 2 * aps, sx128 = 3 * aps;
    static constexpr int sx_floats = 4 * aps * mpad;
    // partial-sum sets per row tile at a flush: stage groups x K slices
    static constexpr int nset = groups * kparts;
    // MMA-warp exchange buffer: [nset-1][8 tiles][NT][4][32 lanes] fp32
    static constexpr int xchg_bytes = (nset - 1) * 8 * NT * 4 * 32 * 4;
};
constexpr int kMaxStages = 8;

struct DecodeParams {
    const uint32_t* qw;       // device layout
    const __half* scales;     // [G,N]
    const __half* zeros;      // [G,N] or null
    const int32_t* g_idx;     // [K] or null
    const float* s_inv;       // [K] or null
    const int32_t* perm;      // [K] or null: X' column k is channel perm[k] (resident X' only)
    const void* X;            // [M,K] activations (read directly when X' is resident)
    void* Y;                  // [M,N]
    unsigned long long* slots;   // split-K partials: [P][8 tiles][NT][4][32] {fp32 bits, flag}
    int M, N, K, group_size, G, out_dtype;
    int KA;                   // K / 64 atoms per band
    int KU;                   // units (2 atoms) per band
    int tiles;                // N / 16
    int units;                // bands * KU
    int base, rem;            // units per CTA: base (+1 for the first rem CTAs)
    int ngs;                  // group rows staged per stage (scale / zero-point box height)
    int stages;               // ring depth (<= kMaxStages)
    int xres;                 // 1: X' and its sums are prepared once per CTA and stay resident
    int off_res;              // byte offset of the resident X' (after the ring and exchange)
    int off_res_s;            // byte offset of the resident sums: [K/32 | K/64 | K/128][sstride]
    int sstride;              // tokens per row of the activation sums
    int off_xchg;             // byte offset of the MMA-warp exchange buffer
    // byte offsets inside one stage
    int off_x, off_xs, off_sx, off_si, off_sc, off_zr, off_gi, off_desc, stage_bytes;
    int ldx;                  // row stride of X in elements (read by the layer-sequence kernel)
    int srow_bytes;           // bytes of one staged scale row: 256 (fp16 x 128), 128 (FP4 bytes)
    const float* sg32;        // staged X': sums of X' over 32 / 64 / 128 channels,
    const float* sg64;        // [segment][8 NT] fp32 (tokens >= M zero), written by
    const float* sg128;       // prep_acts_kernel
    const float* tscale;      // NVFP4 tensor scale (device fp32), else null
};

W4_DEV int unit_begin(const DecodeParams& p, int c) { return c * p.base + min(c, p.rem); }
W4_DEV int cta_of_unit(const DecodeParams& p, int u) {
    const int split = p.rem * (p.base + 1);
    return u < split ? u / (p.base + 1) : p.rem + (u - split) / p.base;
}
W4_DEV int band_tiles(const DecodeParams& p, int band) {
    return min(kTilesPerBand, p.tiles - band * kTilesPerBand);
}

// The parts of a CTA's unit range [u0,u1), one per band it touches, in processing order:
// when the range ends inside a band, that (contributor) part comes first, so its partial
// sums are published early; the whole bands follow, and the first band of the range comes
// last: when the range starts inside it, that part completes the band and has to wait for
// the contributors' sums, which by then (each contributor publishes in its first part)
// are normally out.
struct PartIter {
    int b0, b1;
    int lead;   // 1 when the last band is a contributor part (processed first)
    W4_DEV PartIter(const DecodeParams& p, int u0, int u1) {
        b0 = u0 / p.KU;
        b1 = (u1 - 1) / p.KU;
        lead = (b1 > b0 && u1 < (b1 + 1) * p.KU) ? 1 : 0;
    }
    W4_DEV int count() const { return b1 - b0 + 1; }
    W4_DEV int band(int pi) const {
        if (pi == b1 - b0) return b0;
        if (lead && pi == 0) return b1;
        return b0 + 1 + pi - lead;
    }
};

// Atom range [a0, a0+na) of stage st of the part [ps,pe) of `band`, UPS units per stage.
template <int UPS>
W4_DEV void stage_atoms(const DecodeParams& p, int band, int ps, int pe, int st, int& a0, int& na) {
    const int u = ps + UPS * st;
    const int nu = min(UPS, pe - u);
    a0 = 2 * (u - band * p.KU);
    na = min(2 * nu, p.KA - a0);
}

W4_DEV void store_out(const DecodeParams& p, int m, int n, float v) {
    const size_t idx = (size_t)m * p.N + n;
    if (p.out_dtype == 2) reinterpret_cast<float*>(p.Y)[idx] = v;
    else if (p.out_dtype == 1) reinterpret_cast<__nv_bfloat16*>(p.Y)[idx] = __float2bfloat16_rn(v);
    else reinterpret_cast<__half*>(p.Y)[idx] = __float2half_rn(v);
}

// Shared-memory loads through pointers derived from the dynamic shared array (the
// compiler keeps them after the mbarrier waits, whose asm clobbers memory, and is free to
// schedule them otherwise).
W4_DEV uint32_t ld_u32(const unsigned char* p) { return *reinterpret_cast<const uint32_t*>(p); }
W4_DEV uint32_t ld_u16(const unsigned char* p) { return *reinterpret_cast<const unsigned short*>(p); }
W4_DEV uint4 ld_u128(const unsigned char* p) { return *reinterpret_cast<const uint4*>(p); }
W4_DEV float2 ld_f2(const unsigned char* p) { return *reinterpret_cast<const float2*>(p); }

// Split-K partial words: {fp32 bits (low), flag 1 (high)}, one 64-bit access each.
W4_DEV void slot_put(unsigned long long* a, float v) {
    const unsigned long long w = (1ull << 32) | (unsigned long long)__float_as_uint(v);
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(a), "l"(w) : "memory");
}
W4_DEV unsigned long long slot_get(const unsigned long long* a) {
    unsigned long long w;
    asm volatile("ld.relaxed.gpu.global.b64 %0, [%1];" : "=l"(w) : "l"(a) : "memory");
    return w;
}
W4_DEV void slot_clear(unsigned long long* a) {
    asm volatile("st.relaxed.gpu.global.b64 [%0], %1;" ::"l"(a), "l"(0ull) : "memory");
}

// Wait (bounded) until a published partial word carries its flag; returns its value.
W4_DEV bool slot_wait(const unsigned long long* a, float& v) {
    unsigned long long w = slot_get(a);
    if ((w >> 32) == 0) {
        const uint64_t t0 = globaltimer_ns();
        const uint64_t limit = *(volatile unsigned long long*)&g_w4_wait_limit_ns;
        for (uint32_t it = 1;; ++it) {
            w = slot_get(a);
            if ((w >> 32) != 0) break;
            if ((it & 15u) == 0u) {
                if (globaltimer_ns() - t0 > limit) {
                    atomicOr(&g_w4_error_word, W4_DEVERR_TIMEOUT);
                    return false;
                }
                __nanosleep(64);
            }
        }
    }
    v = __uint_as_float((uint32_t)w);
    return true;
}

// ---------------------------------------------------------------- MMA-warp building blocks
// Biased unpack of one device-layout word (see the layout in w4a16.h): four A-operand
// registers of a 16x16 MMA slice, a[0] = row r0 cols c,c+1; a[1] = row r1 cols c,c+1;
// a[2] = row r0 cols c+8,c+9; a[3] = row r1 cols c+8,c+9, each element o + m*q exactly:
//   fp16: rows r0 (nibbles 0,2,4,6): 1024 + q;  rows r1 (nibbles 1,3,5,7): 1024 + 16 q;
//   bf16: every element 128 + q.
template <bool BF16>
W4_DEV void unpack_biased(uint32_t w, uint32_t (&a)[4]) {
    if constexpr (!BF16) {
        const uint32_t w8 = w >> 8;
        a[0] = and_or(w, 0x000F000Fu, 0x64006400u);
        a[1] = and_or(w, 0x00F000F0u, 0x64006400u);
        a[2] = and_or(w8, 0x000F000Fu, 0x64006400u);
        a[3] = and_or(w8, 0x00F000F0u, 0x64006400u);
    } else {
        a[0] = and_or(w, 0x000F000Fu, 0x43004300u);
        a[1] = and_or(w >> 4, 0x000F000Fu, 0x43004300u);
        a[2] = and_or(w >> 8, 0x000F000Fu, 0x43004300u);
        a[3] = and_or(w >> 12, 0x000F000Fu, 0x43004300u);
    }
}

// Fold constants of one row for one group: sum_k (q - z) X' = (c + bz * S) * mul ... times
// the scale, i.e. acc += sc' * (c + bz * S) with sc' = scale / m and bz = -(o + m z).
struct RowFold {
    float scp, bz;
};

template <bool BF16, bool HI>
W4_DEV RowFold row_fold(uint32_t sc_bits, uint32_t z_bits) {
    const float sc = __half2float(__ushort_as_half((unsigned short)sc_bits));
    const float z = __half2float(__ushort_as_half((unsigned short)z_bits));
    RowFold f;
    if constexpr (BF16) {
        f.scp = sc;
        f.bz = -(128.0f + z);
    } else if constexpr (HI) {
        f.scp = sc * 0.0625f;
        f.bz = -fmaf(16.0f, z, 1024.0f);
    } else {
        f.scp = sc;
        f.bz = -(1024.0f + z);
    }
    return f;
}

// Per-lane constants of an MMA warp.
struct Lane {
    int lane, g8, q;
    int st;                  // token offset of this lane's activation-sum pair
    int xlo[4], xhi[4];      // activation fragment byte offsets of the 16-deep steps
};

// X' is stored [token row][column block][128 B], each 128-byte line swizzled by its row
// (16-byte chunk c at (c ^ (row & 7)) * 16), `rs` bytes per row.  xrows: token rows
// stored; with fewer than 8, lanes of token rows >= M read row M-1 instead (their
// products land in accumulator columns that are never stored).
W4_DEV Lane make_lane(int lane, int xrows, int sstride, int rs) {
    Lane L;
    L.lane = lane;
    L.g8 = lane >> 2;
    L.q = lane & 3;
    L.st = min(2 * L.q, sstride - 2);   // token pairs beyond the stored ones: never stored
    const int row = min(L.g8, xrows - 1);
    // row `row` of a 128B-swizzled line, k pairs 8j+q (b0) and 8j+4+q (b1) of step j
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        L.xlo[j] = row * rs + ((((2 * j) ^ row) & 7) << 4) + 4 * L.q;
        L.xhi[j] = row * rs + ((((2 * j + 1) ^ row) & 7) << 4) + 4 * L.q;
    }
    return L;
}


// What an MMA warp needs about the stage being consumed.
struct StageView {
    const unsigned char* codes;   // the stage's packed tiles: [atom][tile][512 B]
    const unsigned char* x;       // activations X': [column block][token row][128 B swizzled]
    const unsigned char* sx32;    // activation sums over 32 / 64 / 128 channels from the
    const unsigned char* sx64;    // stage's first channel: [segment][sstride] fp32
    const unsigned char* sx128;
    int sstride;
    const unsigned char* sc;      // scale rows: [group row][128] fp16
    const unsigned char* zr;      // zero-point rows, or null (symmetric)
    int tb, a0, gfirst;
    int kin, grow;                // first consumed atom: offset in its group, staged group row
};

// Four 8x8 16-bit matrices from shared memory: lane l gives the address of row l % 8 of
// matrix l / 8, and register i receives matrix i in the MMA fragment order (thread t:
// row t / 4, elements 2 (t % 4) and 2 (t % 4) + 1).
W4_DEV void ldmatrix_x4(uint32_t saddr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(saddr));
}

// B fragments of 16-deep step j for every token tile of a staged X' ([token row][block]
// [128 B], rows Cfg::aps * 128 bytes apart, chunks permuted by row): one ldmatrix.x4 per
// pair of token tiles gives b0, b1 of both (the matrices (tile, k 0-7), (tile, k 8-15)).
template <int NT>
W4_DEV void load_b_frags(const unsigned char* xa, int lane, int j, uint32_t (&b0)[NT], uint32_t (&b1)[NT]) {
    static_assert(NT % 2 == 0, "pairs of token tiles");
    constexpr int RS = Cfg<NT>::aps * 128;
    const int m = lane >> 3, rr = lane & 7;
    const uint32_t base = smem_u32(xa) + (uint32_t)((8 * (m >> 1) + rr) * RS + ((((2 * j + (m & 1)) ^ rr) & 7) << 4));
#pragma unroll
    for (int pp = 0; pp < NT / 2; ++pp) {
        uint32_t r[4];
        ldmatrix_x4(base + (uint32_t)(pp * 16 * RS), r);
        b0[2 * pp] = r[0];
        b1[2 * pp] = r[1];
        b0[2 * pp + 1] = r[2];
        b1[2 * pp + 1] = r[3];
    }
}

// D(16x8, fp32) = A(16x16) * B(16x8), no accumulator input.
template <bool BF16>
W4_DEV void mma_16816_z(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
    if constexpr (BF16) {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
    } else {
        asm volatile(
            "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, "
            "{%4,%5,%6,%7}, {%8,%9}, {%10,%10,%10,%10};"
            : "=f"(d[0]), "=f"(d[1]), "=f"(d[2]), "=f"(d[3])
            : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1), "f"(0.0f));
    }
}

// One 16-deep step of TPW row tiles against NT token tiles; FIRST starts the partial sums.
template <int NT, int TPW, bool BF16, bool FIRST>
W4_DEV void mma_step(const uint32_t (&wj)[TPW], const unsigned char* xa, int xl, int xh, int lane, int j,
                     float (&c)[TPW][NT][4]) {
    uint32_t b0[NT], b1[NT];
    if constexpr (NT >= 2) {
        load_b_frags<NT>(xa, lane, j, b0, b1);
    } else {
        b0[0] = ld_u32(xa + xl);
        b1[0] = ld_u32(xa + xh);
    }
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
        uint32_t af[4];
        unpack_biased<BF16>(wj[tt], af);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            if constexpr (FIRST) mma_16816_z<BF16>(c[tt][nt], af, b0[nt], b1[nt]);
            else mma_16816<BF16>(c[tt][nt], af, b0[nt], b1[nt]);
        }
    }
}

template <int NT>
W4_DEV void load_sums(const unsigned char* sx, int seg, int sstride, const Lane& L, float2 (&S)[NT]) {
#pragma unroll
    for (int nt = 0; nt < NT; ++nt) S[nt] = ld_f2(sx + (seg * sstride + 8 * nt + L.st) * 4);
}

// Fold the partial sums c of one group (staged group row `grow`) into acc:
// acc += sc' * (c + bz * S) per element, with the row's {sc', bz} from its staged fp16
// scale and zero point and S, per token tile, the activation sums of tokens 8nt+2q and
// 8nt+2q+1 over the folded channels.
template <int NT, int TPW, bool BF16>
W4_DEV void fold(const StageView& v, const Lane& L, int t0, int grow, const float2 (&S)[NT],
                 const float (&c)[TPW][NT][4], float (&acc)[TPW][NT][4]) {
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
        const int o0 = (grow * kBandRows + 16 * (t0 + tt) + L.g8) * 2, o1 = o0 + 16;
        const uint32_t sc0 = ld_u16(v.sc + o0), sc1 = ld_u16(v.sc + o1);
        const uint32_t z0 = v.zr ? ld_u16(v.zr + o0) : 0x4800u;   // symmetric: z = 8
        const uint32_t z1 = v.zr ? ld_u16(v.zr + o1) : 0x4800u;
        const RowFold f0 = row_fold<BF16, false>(sc0, z0);
        const RowFold f1 = row_fold<BF16, true>(sc1, z1);
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) {
            acc[tt][nt][0] = fmaf(f0.scp, fmaf(f0.bz, S[nt].x, c[tt][nt][0]), acc[tt][nt][0]);
            acc[tt][nt][1] = fmaf(f0.scp, fmaf(f0.bz, S[nt].y, c[tt][nt][1]), acc[tt][nt][1]);
            acc[tt][nt][2] = fmaf(f1.scp, fmaf(f1.bz, S[nt].x, c[tt][nt][2]), acc[tt][nt][2]);
            acc[tt][nt][3] = fmaf(f1.scp, fmaf(f1.bz, S[nt].y, c[tt][nt][3]), acc[tt][nt][3]);
        }
    }
}

template <int TPW>
W4_DEV uint32_t word_j(const uint4& w, int j) { return j == 0 ? w.x : j == 1 ? w.y : j == 2 ? w.z : w.w; }

template <int NT, int TPW>
W4_DEV void zero_acc(float (&c)[TPW][NT][4]) {
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) c[tt][nt][e] = 0.0f;
}

// Consume atoms [ab, ae) of the stage for row tiles t0..t0+TPW-1 (contiguous groups).
template <int NT, int TPW, bool BF16, int MODE>
W4_DEV void consume(const StageView& v, const Lane& L, int t0, int ab, int ae, int g,
                    float (&acc)[TPW][NT][4]) {
    const unsigned char* wl = v.codes + t0 * 512 + L.lane * 16;
    if constexpr (MODE == kModeHalf) {
        // atoms come in pairs, each pair inside one group (at most apk / 2 pairs per call).
        // Every address below is a per-call pointer plus a compile-time offset.  With one
        // token tile the odd 16-deep steps accumulate into a second register set so
        // consecutive MMAs of a tile do not wait on each other.
        constexpr int CH = NT == 1 ? 2 : 1;
        constexpr int NPR = Cfg<NT>::apk / 2;
        const unsigned char* xb = v.x + ab * 128;
        const unsigned char* xq[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            xq[2 * j] = xb + L.xlo[j];
            xq[2 * j + 1] = xb + L.xhi[j];
        }
        const int wstride = v.tb * 512;
        const unsigned char* wp[2 * NPR];
        wp[0] = v.codes + ab * wstride + t0 * 512 + L.lane * 16;
#pragma unroll
        for (int k = 1; k < 2 * NPR; ++k) wp[k] = wp[k - 1] + wstride;
        const unsigned char* scp = v.sc + (16 * t0 + L.g8) * 2;
        const unsigned char* zrp = v.zr + (16 * t0 + L.g8) * 2;
        const unsigned char* sxp = v.sx128 + ((ab >> 1) * v.sstride + L.st) * 4;
        // staged group row of the first pair and the pair's offset inside its group
        int kin = v.kin;
        int grow = v.grow;
#pragma unroll
        for (int pr = 0; pr < NPR; ++pr) {
            if (ab + 2 * pr >= ae) break;
            uint4 w[2][TPW];
#pragma unroll
            for (int aa = 0; aa < 2; ++aa)
#pragma unroll
                for (int tt = 0; tt < TPW; ++tt) w[aa][tt] = ld_u128(wp[2 * pr + aa] + tt * 512);
            // scale and zero-point bits of rows r0 and r1 of each tile
            uint32_t md[TPW][4];
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
                const int o = grow * 256 + tt * 32;
                md[tt][0] = ld_u16(scp + o);
                md[tt][1] = ld_u16(scp + o + 16);
                md[tt][2] = v.zr ? ld_u16(zrp + o) : 0x4800u;   // symmetric: z = 8
                md[tt][3] = v.zr ? ld_u16(zrp + o + 16) : 0x4800u;
            }
            float c[TPW][NT][4], c2[TPW][NT][4];
#pragma unroll
            for (int aa = 0; aa < 2; ++aa)
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    const int xo = (2 * pr + aa) * 128;
                    uint32_t b0[NT], b1[NT];
                    if constexpr (NT >= 2) {
                        load_b_frags<NT>(xb + xo, L.lane, j, b0, b1);
                    } else {
                        b0[0] = ld_u32(xq[2 * j] + xo);
                        b1[0] = ld_u32(xq[2 * j + 1] + xo);
                    }
                    const int st = 4 * aa + j;
#pragma unroll
                    for (int tt = 0; tt < TPW; ++tt) {
                        uint32_t af[4];
                        unpack_biased<BF16>(word_j<TPW>(w[aa][tt], j), af);
#pragma unroll
                        for (int nt = 0; nt < NT; ++nt) {
                            float (&d)[4] = (CH == 2 && (st & 1)) ? c2[tt][nt] : c[tt][nt];
                            if (st < CH) mma_16816_z<BF16>(d, af, b0[nt], b1[nt]);
                            else mma_16816<BF16>(d, af, b0[nt], b1[nt]);
                        }
                    }
                }
            if constexpr (CH == 2) {
#pragma unroll
                for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e) c[tt][nt][e] += c2[tt][nt][e];
            }
            float2 S[NT];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) S[nt] = ld_f2(sxp + (pr * v.sstride + 8 * nt) * 4);
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
                const RowFold f0 = row_fold<BF16, false>(md[tt][0], md[tt][2]);
                const RowFold f1 = row_fold<BF16, true>(md[tt][1], md[tt][3]);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    acc[tt][nt][0] = fmaf(f0.scp, fmaf(f0.bz, S[nt].x, c[tt][nt][0]), acc[tt][nt][0]);
                    acc[tt][nt][1] = fmaf(f0.scp, fmaf(f0.bz, S[nt].y, c[tt][nt][1]), acc[tt][nt][1]);
                    acc[tt][nt][2] = fmaf(f1.scp, fmaf(f1.bz, S[nt].x, c[tt][nt][2]), acc[tt][nt][2]);
                    acc[tt][nt][3] = fmaf(f1.scp, fmaf(f1.bz, S[nt].y, c[tt][nt][3]), acc[tt][nt][3]);
                }
            }
            kin += 128;
            if (kin >= g) {
                kin -= g;
                ++grow;
            }
        }
    } else {
        // atom by atom; the activation sums accumulate until the fold
        float c[TPW][NT][4];
        zero_acc<NT, TPW>(c);
        float2 S[NT];
#pragma unroll
        for (int nt = 0; nt < NT; ++nt) S[nt] = make_float2(0.0f, 0.0f);
#pragma unroll 1
        for (int a = ab; a < ae; ++a) {
            uint4 w[TPW];
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) w[tt] = ld_u128(wl + (a * v.tb + tt) * 512);
            const unsigned char* xa = v.x + a * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                uint32_t wj[TPW];
#pragma unroll
                for (int tt = 0; tt < TPW; ++tt) wj[tt] = word_j<TPW>(w[tt], j);
                mma_step<NT, TPW, BF16, false>(wj, xa, L.xlo[j], L.xhi[j], L.lane, j, c);
                if constexpr (MODE == kModeG32) {
                    if (j & 1) {
                        float2 S32[NT];
                        load_sums<NT>(v.sx32, 2 * a + (j >> 1), v.sstride, L, S32);
                        fold<NT, TPW, BF16>(v, L, t0, 2 * a + (j >> 1), S32, c, acc);
                        zero_acc<NT, TPW>(c);
                    }
                }
            }
            if constexpr (MODE == kModeAtom) {
                float2 S64[NT];
                load_sums<NT>(v.sx64, a, v.sstride, L, S64);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    S[nt].x += S64[nt].x;
                    S[nt].y += S64[nt].y;
                }
                if ((64 * (v.a0 + a + 1)) % g == 0 || a == ae - 1) {
                    fold<NT, TPW, BF16>(v, L, t0, (64 * (v.a0 + a)) / g - v.gfirst, S, c, acc);
                    zero_acc<NT, TPW>(c);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) S[nt] = make_float2(0.0f, 0.0f);
                }
            }
        }
    }
}

// FP4 weights: the E2M1 codes become exact fp16 values (w4f::unpack_fp4); the MMA sums
// each scale block's products and the block's scale multiplies that partial in fp32.
// Scale of one staged block-scale byte: E4M3 (NVFP4) or 2^(byte - 127) (MXFP4; the
// byte 0, 2^-127, reads as 0: such a block's weights are below 2^-124).
template <int MODE>
W4_DEV float fp4_block_scale(uint32_t byte) {
    if constexpr (MODE == kModeNvfp4) return w4f::e4m3_to_f32(byte);
    else return __int_as_float(byte << 23);
}

// gs: the NVFP4 tensor scale, folded into every block scale (1 for MXFP4).
template <int NT, int TPW, int MODE>
W4_DEV void consume_fp4(const StageView& v, const Lane& L, int t0, int ab, int ae, float gs,
                        float (&acc)[TPW][NT][4]) {
    constexpr int B = MODE == kModeNvfp4 ? 16 : 32;   // channels per scale block
    const unsigned char* wl = v.codes + t0 * 512 + L.lane * 16;
#pragma unroll 1
    for (int a = ab; a < ae; ++a) {
        uint4 w[TPW];
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) w[tt] = ld_u128(wl + (a * v.tb + tt) * 512);
        const unsigned char* xa = v.x + a * 128;
        float c[TPW][NT][4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            uint32_t b0[NT], b1[NT];
            if constexpr (NT >= 2) {
                load_b_frags<NT>(xa, L.lane, j, b0, b1);
            } else {
                b0[0] = ld_u32(xa + L.xlo[j]);
                b1[0] = ld_u32(xa + L.xhi[j]);
            }
            const bool first = B == 16 || (j & 1) == 0;
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
                uint32_t af[4];
                w4f::unpack_fp4(word_j<TPW>(w[tt], j), af);
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (first) mma_16816_z<false>(c[tt][nt], af, b0[nt], b1[nt]);
                    else mma_16816<false>(c[tt][nt], af, b0[nt], b1[nt]);
                }
            }
            if (B == 16 || (j & 1)) {
                // the block's staged scale row, rows r0 / r1 of each tile
                const unsigned char* srow = v.sc + ((64 * (v.a0 + a) + 16 * j) / B - v.gfirst) * 128;
#pragma unroll
                for (int tt = 0; tt < TPW; ++tt) {
                    const int r0 = 16 * (t0 + tt) + L.g8;
                    const float s0 = fp4_block_scale<MODE>(srow[r0]) * gs;
                    const float s1 = fp4_block_scale<MODE>(srow[r0 + 8]) * gs;
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        acc[tt][nt][0] = fmaf(s0, c[tt][nt][0], acc[tt][nt][0]);
                        acc[tt][nt][1] = fmaf(s0, c[tt][nt][1], acc[tt][nt][1]);
                        acc[tt][nt][2] = fmaf(s1, c[tt][nt][2], acc[tt][nt][2]);
                        acc[tt][nt][3] = fmaf(s1, c[tt][nt][3], acc[tt][nt][3]);
                    }
                }
            }
        }
    }
}

// Act-order: every input channel k has its own group g_idx[k]; each weight is dequantised
// to fp16 (q - z[g_idx[k], n]) * scale[g_idx[k], n] before the MMA (fp16 activations only).
template <int NT, int TPW>
W4_DEV void consume_gidx(const StageView& v, const DecodeParams& p, const Lane& L, int band, int t0,
                         int ab, int ae, const unsigned char* gis, float (&acc)[TPW][NT][4]) {
    const unsigned char* wl = v.codes + t0 * 512 + L.lane * 16;
#pragma unroll 1
    for (int a = ab; a < ae; ++a) {
        const unsigned char* xa = v.x + a * 128;
#pragma unroll 1
        for (int j = 0; j < 4; ++j) {
            const int kk = 64 * a + 16 * j + 2 * L.q;
            int gk[4] = {(int)ld_u32(gis + 4 * kk), (int)ld_u32(gis + 4 * (kk + 1)),
                         (int)ld_u32(gis + 4 * (kk + 8)), (int)ld_u32(gis + 4 * (kk + 9))};
#pragma unroll
            for (int e = 0; e < 4; ++e)
                if (gk[e] < 0 || gk[e] >= p.G) {
                    atomicOr(&g_w4_error_word, W4_DEVERR_GIDX);
                    gk[e] = 0;
                }
            uint32_t b0[NT], b1[NT];
            if constexpr (NT >= 2) {
                load_b_frags<NT>(xa, L.lane, j, b0, b1);
            } else {
                b0[0] = ld_u32(xa + L.xlo[j]);
                b1[0] = ld_u32(xa + L.xhi[j]);
            }
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt) {
                if (t0 + tt >= v.tb) continue;   // rows beyond N: no metadata to gather
                const uint32_t wv = word_j<TPW>(ld_u128(wl + (a * v.tb + tt) * 512), j);
                const int nr0 = band * kBandRows + 16 * (t0 + tt) + L.g8, nr1 = nr0 + 8;
                uint32_t af[4];
#pragma unroll
                for (int r = 0; r < 4; ++r) {
                    // register r holds nibbles r and r+4: rows r0/r1 (r odd), columns
                    // c,c+1 (r < 2) or c+8,c+9 (r >= 2)
                    const int row = (r & 1) ? nr1 : nr0;
                    const int kl = (r & 2) ? 2 : 0;
                    const float qlo = (float)((wv >> (4 * r)) & 0xF);
                    const float qhi = (float)((wv >> (4 * (r + 4))) & 0xF);
                    const __half z_lo = p.zeros ? __ldg(p.zeros + (size_t)gk[kl] * p.N + row) : __float2half_rn(8.0f);
                    const __half z_hi = p.zeros ? __ldg(p.zeros + (size_t)gk[kl + 1] * p.N + row) : __float2half_rn(8.0f);
                    const __half2 ss = __halves2half2(__ldg(p.scales + (size_t)gk[kl] * p.N + row),
                                                      __ldg(p.scales + (size_t)gk[kl + 1] * p.N + row));
                    af[r] = h2_as_u32(__hmul2(__hsub2(__floats2half2_rn(qlo, qhi), __halves2half2(z_lo, z_hi)), ss));
                }
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) mma_16816<false>(acc[tt][nt], af, b0[nt], b1[nt]);
            }
        }
    }
}

// ---------------------------------------------------------------- prepared activations
// X' = X * s_inv rounded to the activation type (a plain copy without s_inv) and its sums
// over every 32, 64 and 128 channels, once per GEMM, for the decode kernel's staged
// activations: X' [M, K] with the 16-byte chunks of every 128-byte block permuted by the
// row (chunk c of row m at c ^ (m & 7), the bank-conflict-free order the MMA warps read),
// so that one tensor copy per stage lands it in shared memory as [row][block][128 B];
// sums [segment][mpad], rows M..mpad-1 zero.  Thread t takes 8-channel chunk t % (K/8)
// of token row t / (K/8): consecutive lanes hold consecutive chunks of one row, so the
// sums are warp shuffles.
template <bool BF16>
__global__ void prep_acts_kernel(const void* __restrict__ X, const float* __restrict__ s_inv, int M, int K,
                                 int mpad, void* __restrict__ Xp, float* __restrict__ s32,
                                 float* __restrict__ s64, float* __restrict__ s128) {
    // launched with programmatic dependent launch: the decode kernel after it may start
    // its prologue and weight copies at once (it waits for this grid before reading X');
    // X itself may come from the kernel before
    pdl_launch_dependents();
    pdl_wait();
    const int cpt = K / 8;
    const size_t t = blockIdx.x * (size_t)blockDim.x + threadIdx.x;
    const int lane = threadIdx.x & 31;
    const bool valid = t < (size_t)mpad * cpt;
    const int m = valid ? (int)(t / cpt) : 0, c = valid ? (int)(t % cpt) : 0;
    float s = 0.0f;
    if (valid && m < M) {
        uint4 v = reinterpret_cast<const uint4*>(X)[(size_t)m * cpt + c];
        uint32_t w[4] = {v.x, v.y, v.z, v.w};
        if (s_inv) {
            const float4 a = __ldg(reinterpret_cast<const float4*>(s_inv) + 2 * c);
            const float4 b = __ldg(reinterpret_cast<const float4*>(s_inv) + 2 * c + 1);
            const float sv[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = unpack2<BF16>(w[i]);
                w[i] = pack2<BF16>(__fmul_rn(f.x, sv[2 * i]), __fmul_rn(f.y, sv[2 * i + 1]));
            }
        }
        const int blk = c >> 3, ch = c & 7;
        reinterpret_cast<uint4*>(Xp)[(size_t)m * cpt + 8 * blk + (ch ^ (m & 7))] = make_uint4(w[0], w[1], w[2], w[3]);
        float2 f[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = unpack2<BF16>(w[i]);
        s = ((f[0].x + f[0].y) + (f[1].x + f[1].y)) + ((f[2].x + f[2].y) + (f[3].x + f[3].y));
    }
    // groups of 4 / 8 / 16 consecutive chunks are aligned to 32 / 64 / 128 channels (K is a
    // multiple of 64; the 128-channel sums are only read when K is a multiple of 128)
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (valid && (lane & 3) == 0) s32[(c >> 2) * mpad + m] = s;
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    if (valid && (lane & 7) == 0) s64[(c >> 3) * mpad + m] = s;
    s += __shfl_xor_sync(0xffffffffu, s, 8);
    if (valid && (lane & 15) == 0 && (c >> 4) < K / 128) s128[(c >> 4) * mpad + m] = s;
}

// Resident activations (one token tile, small M*K): X' = X * s_inv for the whole of K and
// its sums over every 32, 64 and 128 channels, prepared once per CTA by the warps
// [w0, w0 + nw) straight from global memory.  X' keeps the per-stage layout, M rows per
// 64-channel block; sums are [segment][sstride].  Consecutive lanes take consecutive
// 8-channel chunks, so the sums are warp shuffles; a lane takes its chunk for every token
// (M <= 8 here), loading the chunk's s_inv once and all M activation chunks together.
// The 8-channel chunks of X' that the units [u0, u1) read: the whole row when the range
// holds a band's worth of units, else the K units of the range (one run, or two when
// the range crosses into the next band), rounded out to 16 chunks and clipped to K.
W4_DEV void prep_ranges(const DecodeParams& p, int u0, int u1, int& ca0, int& ca1, int& cb0, int& cb1) {
    const int cpt = p.K / 8;
    ca0 = ca1 = cb0 = cb1 = 0;
    if (u0 >= u1) return;
    if (u1 - u0 >= p.KU) {
        ca1 = cpt;
        return;
    }
    const int lo = u0 % p.KU, hi = (u1 - 1) % p.KU;
    if (lo <= hi) {
        ca0 = 16 * lo;
        ca1 = min(16 * (hi + 1), cpt);
    } else {
        ca0 = 16 * lo;
        ca1 = cpt;
        cb1 = min(16 * (hi + 1), cpt);
    }
}

// COHERENT: X was written earlier in the same launch by other CTAs (the layer-sequence
// kernel), so it is read through L2 (ld.global.cg), with rows p.ldx elements apart.
// Only the chunks [ca0, ca1) and [cb0, cb1) are prepared: the input channels of the CTA's
// own units (multiples of 16 chunks, i.e. of 128 channels, so that the 32-, 64- and
// 128-channel sums of a warp's lanes never straddle the two ranges).
template <bool BF16, bool PERM, bool COHERENT = false>
W4_DEV void prep_resident(const DecodeParams& p, const void* X, unsigned char* xr, float* sr, int w,
                          int nw, int lane, int ca0, int ca1, int cb0, int cb1) {
    const int cpt = p.K / 8;                       // chunks per token
    const int rpt = COHERENT ? p.ldx / 8 : cpt;    // chunks between consecutive token rows
    const int ss = p.sstride;
    float* s32 = sr;
    float* s64 = s32 + (p.K / 32) * ss;
    float* s128 = s64 + (p.K / 64) * ss;
    const uint4* x4 = reinterpret_cast<const uint4*>(X);
    // lanes walk the first range, then (from the next multiple of 16 lanes) the second
    const int na = ca1 - ca0, nb0 = (na + 15) / 16 * 16, nv = nb0 + (cb1 - cb0);
    for (int base = 32 * w; base < nv; base += 32 * nw) {
        const int vi = base + lane;
        const bool valid = vi < na || (vi >= nb0 && vi < nv);
        const int c = vi < na ? ca0 + vi : cb0 + (vi - nb0);
        float sv[8];
#pragma unroll
        for (int i = 0; i < 8; ++i) sv[i] = 1.0f;
        uint4 v[8];
        if constexpr (PERM) {
            // act-order weights packed with contiguous groups: gather channel perm[k] into
            // column k (an entry outside [0, K) is reported and reads channel 0)
            int src[8] = {0, 0, 0, 0, 0, 0, 0, 0};
            if (valid) {
                const int4 p0 = __ldg(reinterpret_cast<const int4*>(p.perm) + 2 * c);
                const int4 p1 = __ldg(reinterpret_cast<const int4*>(p.perm) + 2 * c + 1);
                src[0] = p0.x; src[1] = p0.y; src[2] = p0.z; src[3] = p0.w;
                src[4] = p1.x; src[5] = p1.y; src[6] = p1.z; src[7] = p1.w;
#pragma unroll
                for (int i = 0; i < 8; ++i)
                    if (src[i] < 0 || src[i] >= p.K) {
                        atomicOr(&g_w4_error_word, W4_DEVERR_GIDX);
                        src[i] = 0;
                    }
                if (p.s_inv) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) sv[i] = __ldg(p.s_inv + src[i]);
                }
            }
            const unsigned short* xh = reinterpret_cast<const unsigned short*>(X);
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                uint32_t h[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                if (valid && m < p.M) {
#pragma unroll
                    for (int i = 0; i < 8; ++i) h[i] = xh[(size_t)m * p.K + src[i]];
                }
                v[m] = make_uint4(h[0] | (h[1] << 16), h[2] | (h[3] << 16), h[4] | (h[5] << 16), h[6] | (h[7] << 16));
            }
        } else {
            if (p.s_inv && valid) {
                const float4 s0 = __ldg(reinterpret_cast<const float4*>(p.s_inv) + 2 * c);
                const float4 s1 = __ldg(reinterpret_cast<const float4*>(p.s_inv) + 2 * c + 1);
                sv[0] = s0.x; sv[1] = s0.y; sv[2] = s0.z; sv[3] = s0.w;
                sv[4] = s1.x; sv[5] = s1.y; sv[6] = s1.z; sv[7] = s1.w;
            }
#pragma unroll
            for (int m = 0; m < 8; ++m) {
                if constexpr (COHERENT)
                    v[m] = (valid && m < p.M) ? __ldcg(x4 + (size_t)m * rpt + c) : make_uint4(0u, 0u, 0u, 0u);
                else
                    v[m] = (valid && m < p.M) ? x4[(size_t)m * rpt + c] : make_uint4(0u, 0u, 0u, 0u);
            }
        }
        const int blk = c >> 3, ch = c & 7;
#pragma unroll
        for (int m = 0; m < 8; ++m) {
            if (m >= p.M) break;
            float s = 0.0f;
            if (valid) {
                uint32_t wv[4] = {v[m].x, v[m].y, v[m].z, v[m].w};
                if (p.s_inv) {
#pragma unroll
                    for (int i = 0; i < 4; ++i) {
                        const float2 f = unpack2<BF16>(wv[i]);
                        wv[i] = pack2<BF16>(__fmul_rn(f.x, sv[2 * i]), __fmul_rn(f.y, sv[2 * i + 1]));
                    }
                }
                *reinterpret_cast<uint4*>(xr + m * (p.K / 64 * 128) + blk * 128 + ((ch ^ (m & 7)) << 4)) =
                    make_uint4(wv[0], wv[1], wv[2], wv[3]);
                float2 f[4];
#pragma unroll
                for (int i = 0; i < 4; ++i) f[i] = unpack2<BF16>(wv[i]);
                s = ((f[0].x + f[0].y) + (f[1].x + f[1].y)) + ((f[2].x + f[2].y) + (f[3].x + f[3].y));
            }
            // groups of 4 / 8 / 16 consecutive chunks are aligned to 32 / 64 / 128 channels
            // (K is a multiple of 64; the 128-channel sums are only read when K is a
            // multiple of 128)
            s += __shfl_xor_sync(0xffffffffu, s, 1);
            s += __shfl_xor_sync(0xffffffffu, s, 2);
            if (valid && (lane & 3) == 0) s32[(c >> 2) * ss + m] = s;
            s += __shfl_xor_sync(0xffffffffu, s, 4);
            if (valid && (lane & 7) == 0) s64[(c >> 3) * ss + m] = s;
            s += __shfl_xor_sync(0xffffffffu, s, 8);
            if (valid && (lane & 15) == 0 && (c >> 4) < p.K / 128) s128[(c >> 4) * ss + m] = s;
        }
    }
}

// ---------------------------------------------------------------- end of a part
// Combine, then store, publish or complete the band's sums.  Slot entry of (tile t, token
// tile nt, element e, lane) is ((t * NT + nt) * 4 + e) * 32 + lane.

// Slot index of entry x of a band's shares, entries ordered by (channel in the band, token).
template <int NT>
W4_DEV int share_slot(int x, int M) {
    const int m = x % M, nl = x / M;
    const int r = nl & 15;
    return (((nl >> 4) * NT + (m >> 3)) * 4 + 2 * (r >> 3) + (m & 1)) * 32 + 4 * (r & 7) + ((m & 7) >> 1);
}

// MMA thread mt of nthr: for each entry x = mt, mt + nthr, ... of the band, xc[slot] = the
// sum of the shares CTAs [c_first, cta) published, in CTA order.  With several token
// tiles a thread takes 4 of its entries at a time from 2 contributors at a time; with
// one, one entry from up to 8 contributors: up to 8 loads are in flight either way.
// False on a timed-out wait.
template <int NT>
W4_DEV bool sum_shares(const DecodeParams& p, float* xc, int band, int c_first, int cta, int mt, int nthr) {
    constexpr int kSlot = kTilesPerBand * NT * 4 * 32;
    // up to 8 loads in flight: with one token tile a band has few entries and often 4-8
    // contributors; with more tiles, thousands of entries
    constexpr int E = NT == 1 ? 1 : 4, CB = NT == 1 ? 8 : 2;   // entries, contributors per round
    const int n_ent = band_tiles(p, band) * 16 * p.M;
    for (int x0 = mt; x0 < n_ent; x0 += E * nthr) {
        int j[E];
        float tot[E];
#pragma unroll
        for (int e = 0; e < E; ++e) {
            const int x = x0 + e * nthr;
            j[e] = x < n_ent ? share_slot<NT>(x, p.M) : -1;
            tot[e] = 0.0f;
        }
        for (int c0 = c_first; c0 < cta; c0 += CB) {
            unsigned long long v[E][CB];
#pragma unroll
            for (int e = 0; e < E; ++e)
#pragma unroll
                for (int b = 0; b < CB; ++b)
                    v[e][b] = (j[e] >= 0 && c0 + b < cta) ? slot_get(p.slots + (size_t)(c0 + b) * kSlot + j[e]) : 0ull;
#pragma unroll
            for (int e = 0; e < E; ++e)
#pragma unroll
                for (int b = 0; b < CB; ++b) {
                    if (j[e] < 0 || c0 + b >= cta) continue;
                    unsigned long long* a = p.slots + (size_t)(c0 + b) * kSlot + j[e];
                    float val = __uint_as_float((uint32_t)v[e][b]);
                    if ((v[e][b] >> 32) == 0 && !slot_wait(a, val)) return false;
                    tot[e] += val;
                    slot_clear(a);
                }
        }
#pragma unroll
        for (int e = 0; e < E; ++e)
            if (j[e] >= 0) xc[j[e]] = tot[e];
    }
    return true;
}

template <int NT, int TPW>
W4_DEV void combine_sets(unsigned char* xchg, int set, int t0, const Lane& L, float (&acc)[TPW][NT][4]) {
    using C = Cfg<NT>;
    if constexpr (C::nset > 1) {
        float* xc = reinterpret_cast<float*>(xchg);
        constexpr int kSet = 8 * NT * 4 * 32;
        if (set > 0) {
#pragma unroll
            for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
                for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                    for (int e = 0; e < 4; ++e)
                        xc[(set - 1) * kSet + (((t0 + tt) * NT + nt) * 4 + e) * 32 + L.lane] = acc[tt][nt][e];
        }
        named_bar_sync(1, 32 * C::mma_warps);
        if (set == 0) {
#pragma unroll
            for (int k = 1; k < C::nset; ++k)
#pragma unroll
                for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            acc[tt][nt][e] += xc[(k - 1) * kSet + (((t0 + tt) * NT + nt) * 4 + e) * 32 + L.lane];
        }
        named_bar_sync(2, 32 * C::mma_warps);
    }
}

template <int NT, int TPW>
W4_DEV void store_rows(const DecodeParams& p, int band, int t0, const Lane& L, const float (&acc)[TPW][NT][4]) {
    const int tb = band_tiles(p, band);
#pragma unroll
    for (int tt = 0; tt < TPW; ++tt) {
        if (t0 + tt >= tb) continue;
        const int n0 = band * kBandRows + 16 * (t0 + tt) + L.g8;
#pragma unroll
        for (int nt = 0; nt < NT; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = 8 * nt + 2 * L.q + (e & 1);
                if (m < p.M) store_out(p, m, n0 + ((e >> 1) << 3), acc[tt][nt][e]);
            }
    }
}

// A part that does not complete its band (set-0 threads, after combine_sets): a whole band
// is stored; a contributor part publishes this CTA's share into its slots.
template <int NT, int TPW>
W4_DEV void flush_part(const DecodeParams& p, int band, int pe, int cta, int t0, const Lane& L,
                       const float (&acc)[TPW][NT][4]) {
    constexpr int kSlot = kTilesPerBand * NT * 4 * 32;
    const int tb = band_tiles(p, band);
    if (pe < (band + 1) * p.KU) {
        unsigned long long* base = p.slots + (size_t)cta * kSlot;
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt) {
            if (t0 + tt >= tb) continue;
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    if (8 * nt + 2 * L.q + (e & 1) < p.M)
                        slot_put(base + (((t0 + tt) * NT + nt) * 4 + e) * 32 + L.lane, acc[tt][nt][e]);
        }
        return;
    }
    store_rows<NT, TPW>(p, band, t0, L, acc);
}

// The CTA's last part holds the band's last unit and started inside the band: add the
// contributors' shares (CTA order) before this CTA's own, then store.  Runs after the part
// loop, on every MMA warp (named barriers on the shared path).
template <int NT, int TPW>
W4_DEV void complete_band(const DecodeParams& p, unsigned char* smem, unsigned char* xchg, volatile int* s_abort,
                          int band, int cta, int set, int t0, const Lane& L, bool aborted,
                          float (&acc)[TPW][NT][4]) {
    using C = Cfg<NT>;
    const int tb = band_tiles(p, band);
    const int c_first = cta_of_unit(p, band * p.KU);
    // the MMA threads share the band's entries, summing the contributors' shares into a
    // slot-layout buffer (the exchange buffer, or with a single set the first ring stage,
    // idle once every MMA warp is past the last stage); set 0 adds them
    float* xc = reinterpret_cast<float*>(C::nset > 1 ? xchg : smem);
    if constexpr (C::nset == 1) named_bar_sync(1, 32 * C::mma_warps);
    const int mt = threadIdx.x - 32 * (1 + C::xw);
    if (!aborted && !sum_shares<NT>(p, xc, band, c_first, cta, mt, 32 * C::mma_warps)) *s_abort = 1;
    named_bar_sync(1, 32 * C::mma_warps);
    if (set == 0) {
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int j = (((t0 + tt) * NT + nt) * 4 + e) * 32 + L.lane;
                    if (t0 + tt < tb && 8 * nt + 2 * L.q + (e & 1) < p.M) acc[tt][nt][e] = xc[j] + acc[tt][nt][e];
                }
    }
    named_bar_sync(2, 32 * C::mma_warps);
    if (set > 0 || aborted || *s_abort) return;
    store_rows<NT, TPW>(p, band, t0, L, acc);
}

// ---------------------------------------------------------------- the kernel
template <int UPS>
W4_DEV int total_stages(const DecodeParams& p, const PartIter& it, int u0, int u1) {
    int n = 0;
    for (int pi = 0; pi < it.count(); ++pi) {
        const int band = it.band(pi);
        const int ps = max(u0, band * p.KU), pe = min(u1, (band + 1) * p.KU);
        n += (pe - ps + UPS - 1) / UPS;
    }
    return n;
}

// Staged activations of a stage: the prepared X' box ([8*NT rows][aps blocks][128 B],
// rows >= M and blocks beyond K zero-filled) and, unless act-order folds the scales into
// the weights, the sums over its 32-, 64- and 128-channel segments ([segment][8*NT]).
template <int NT, bool GIDX>
W4_DEV uint32_t staged_act_bytes(int na) {
    using C = Cfg<NT>;
    return C::aps * C::mpad * 128 + (GIDX ? 0 : (2 * na + na + (na + 1) / 2) * C::mpad * 4);
}

template <int NT, bool GIDX>
W4_DEV void load_staged_acts(const DecodeParams& p, unsigned char* st, const CUtensorMap* tmap_x, int a0, int na,
                             uint64_t* bar) {
    using C = Cfg<NT>;
    tma_load_3d(st + p.off_x, tmap_x, 0, a0, 0, bar);
    if constexpr (!GIDX) {
        unsigned char* sx = st + p.off_sx;
        bulk_g2s(sx + C::sx32 * C::mpad * 4, p.sg32 + (size_t)(2 * a0) * C::mpad, 2 * na * C::mpad * 4, bar);
        bulk_g2s(sx + C::sx64 * C::mpad * 4, p.sg64 + (size_t)a0 * C::mpad, na * C::mpad * 4, bar);
        bulk_g2s(sx + C::sx128 * C::mpad * 4, p.sg128 + (size_t)(a0 / 2) * C::mpad, (na + 1) / 2 * C::mpad * 4, bar);
    }
}

// Ring position: slot and phase parity of consecutive stages.
struct Ring {
    int s = 0, ph = 0;
    W4_DEV void next(int S) {
        if (++s == S) {
            s = 0;
            ph ^= 1;
        }
    }
};

template <int NT, bool BF16, int MODE, bool PERM>
__global__ void __launch_bounds__(Cfg<NT>::threads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_sc,
                  const __grid_constant__ CUtensorMap tmap_zr, const DecodeParams p) {
    using C = Cfg<NT>;
    constexpr bool GIDX = MODE == kModeGidx;
    constexpr int UPS = C::aps / 2;   // units per stage
    const int S = p.stages;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    unsigned char* xchg = smem + p.off_xchg;
    uint64_t* full = reinterpret_cast<uint64_t*>(xchg + C::xchg_bytes);
    uint64_t* empty = full + kMaxStages;
    volatile int* s_abort = reinterpret_cast<volatile int*>(empty + kMaxStages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    const int u0 = unit_begin(p, cta), u1 = unit_begin(p, cta + 1);
    const int g = p.group_size;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::stage_warps);
        }
        *s_abort = 0;
        fence_mbar_init();
    }
    // resident activation sums of tokens >= M are never written: start from zero (staged
    // X' and sums arrive with rows >= M zero)
    if (p.xres) {
        const int words = (p.K / 32 + p.K / 64 + p.K / 128) * p.sstride;
        for (int i = threadIdx.x; i < words; i += C::threads)
            reinterpret_cast<float*>(smem + p.off_res_s)[i] = 0.0f;
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
    if (u0 >= u1) return;
    const PartIter it(p, u0, u1);

    if (warp == 0) {
        // ------------------------------------------------------------ producer
        // lane 0 arms the stage's barrier and issues one copy per operand: the codes
        // (a contiguous run of the band), the scale and zero-point rows (2-D boxes) or the
        // g_idx slice and, with staged activations, the prepared X' (3-D box: 8*NT token
        // rows x the stage's column blocks, rows >= M and blocks beyond K zero-filled) and
        // its three slices of sums.  The read-only weight operands of the first stages go
        // out before pdl_wait(), the activations (written by the preparation kernel just
        // before) after it.
        const uint64_t policy = policy_evict_first();
        const int total = total_stages<UPS>(p, it, u0, u1);
        const int pro = min(S, total);
        Ring r;
        int i = 0;
        bool abort = false;
        for (int pi = 0; pi < it.count() && !abort; ++pi) {
            const int band = it.band(pi);
            const int ps = max(u0, band * p.KU), pe = min(u1, (band + 1) * p.KU);
            const int tb = band_tiles(p, band);
            for (int stg = 0; UPS * stg < pe - ps; ++stg, ++i, r.next(S)) {
                int a0, na;
                stage_atoms<UPS>(p, band, ps, pe, stg, a0, na);
                if (i >= S) {
                    int ok = 1;
                    if (lane == 0) ok = (!*s_abort && mbar_wait(&empty[r.s], r.ph ^ 1)) ? 1 : 0;
                    ok = __shfl_sync(0xffffffffu, ok, 0);
                    if (!ok) {
                        if (lane == 0) *s_abort = 1;
                        abort = true;
                        break;
                    }
                }
                unsigned char* st = smem + r.s * p.stage_bytes;
                const int g_first = GIDX ? 0 : (64 * a0) / g;
                if (lane == 0) {
                    // stage descriptor for the consumers: {a0, na, tiles, first group row}
                    // and, for each K slice, the offset of its first atom in its group and
                    // its staged group row
                    int kg[8] = {0, 0, 0, 0, 0, 0, 0, 0};
                    if (!GIDX) {
#pragma unroll
                        for (int k = 0; k < C::kparts; ++k) {
                            const int off = 64 * a0 - g_first * g + 64 * C::apk * k;
                            kg[2 * k + 1] = off / g;
                            kg[2 * k] = off - kg[2 * k + 1] * g;
                        }
                    }
                    int4* desc = reinterpret_cast<int4*>(st + p.off_desc);
                    desc[0] = make_int4(a0, na, tb, g_first);
                    desc[1] = make_int4(kg[0], kg[1], kg[2], kg[3]);
                    desc[2] = make_int4(kg[4], kg[5], kg[6], kg[7]);
                    uint32_t bytes = na * tb * 512;
                    if (!p.xres) bytes += staged_act_bytes<NT, GIDX>(na);
                    if (GIDX) bytes += na * 256;
                    else bytes += p.ngs * (MODE == kModeNvfp4 || MODE == kModeMxfp4 ? 128 : 256) * (p.zeros ? 2 : 1);
                    mbar_arrive_expect_tx(&full[r.s], bytes);
                    bulk_g2s_hint(st, p.qw + 128 * ((size_t)kTilesPerBand * p.KA * band + (size_t)a0 * tb),
                                  na * tb * 512, &full[r.s], policy);
                    if (GIDX) {
                        bulk_g2s(st + p.off_gi, p.g_idx + 64 * a0, na * 256, &full[r.s]);
                    } else {
                        tma_load_2d(st + p.off_sc, &tmap_sc, band * kBandRows, g_first, &full[r.s]);
                        if (p.zeros) tma_load_2d(st + p.off_zr, &tmap_zr, band * kBandRows, g_first, &full[r.s]);
                    }
                    if (i >= S && !p.xres) load_staged_acts<NT, GIDX>(p, st, &tmap_x, a0, na, &full[r.s]);
                }
                if (i == pro - 1 && !p.xres) {
                    // the activations of the first stages, once the preceding grid is done
                    pdl_wait();
                    int k = 0;
                    for (int pj = 0; pj < it.count() && k < pro; ++pj) {
                        const int bj = it.band(pj);
                        const int qs = max(u0, bj * p.KU), qe = min(u1, (bj + 1) * p.KU);
                        for (int sj = 0; UPS * sj < qe - qs && k < pro; ++sj, ++k) {
                            int aj, nj;
                            stage_atoms<UPS>(p, bj, qs, qe, sj, aj, nj);
                            unsigned char* sk = smem + k * p.stage_bytes;
                            if (lane == 0) load_staged_acts<NT, GIDX>(p, sk, &tmap_x, aj, nj, &full[k]);
                        }
                    }
                }
            }
        }
        // On abort, wait (bounded) for the copies already issued before leaving (an abort
        // can only happen at i >= S, after every prologue copy went out).
        if (abort && lane == 0) {
            Ring q;
            for (int k = 0; k < i; ++k, q.next(S))
                if (k >= i - S) (void)mbar_wait(&full[q.s], q.ph);
        }
        __syncwarp();
    } else {
    if constexpr (NT == 1) {   // (the host sets xres for one token tile only)
    if (p.xres) {
        // ------------------------------------------------------------ resident X'
        pdl_wait();   // X may come from the preceding kernel
        int ca0, ca1, cb0, cb1;
        prep_ranges(p, u0, u1, ca0, ca1, cb0, cb1);
        prep_resident<BF16, PERM>(p, p.X, smem + p.off_res, reinterpret_cast<float*>(smem + p.off_res_s),
                                  warp - 1, C::warps - 1, lane, ca0, ca1, cb0, cb1);
        named_bar_sync(3, C::threads - 32);
    }
    }
    {
        // ------------------------------------------------------------ MMA warps
        pdl_wait();   // before any store to Y or the workspace
        constexpr int TPW = C::tpw;
        const int cw = warp - 1 - C::xw;
        const int grp = cw / C::stage_warps, ws = cw % C::stage_warps;   // stage group, warp in it
        const int kp = ws / C::tsets;                  // K slice of the stage
        const int t0 = TPW * (ws % C::tsets);          // first row tile
        const int set = grp * C::kparts + kp;          // partial-sum set at a flush
        const int xrows = p.xres ? p.M : C::mpad;   // staged X' rows >= M are zero
        const int sstride = p.xres ? p.sstride : C::mpad;
        const Lane L = make_lane(lane, xrows, sstride, p.xres ? p.K / 64 * 128 : C::aps * 128);
        float acc[TPW][NT][4];
        zero_acc<NT, TPW>(acc);
        bool aborted = false;
        Ring r;
        int i = 0;
        for (int pi = 0; pi < it.count(); ++pi) {
            const int band = it.band(pi);
            const int ps = max(u0, band * p.KU), pe = min(u1, (band + 1) * p.KU);
            const int tb = band_tiles(p, band);
            for (int stg = 0; UPS * stg < pe - ps; ++stg, ++i, r.next(S)) {
                if ((i % C::groups) != grp) continue;   // the other group's stage
                if (!aborted) {
                    aborted = *s_abort || !mbar_wait(&full[r.s], r.ph);
                    if (aborted) *s_abort = 1;
                }
                unsigned char* st = smem + r.s * p.stage_bytes;
                const int4 d0 = *reinterpret_cast<const int4*>(st + p.off_desc);
                const int2 kg = *reinterpret_cast<const int2*>(st + p.off_desc + 16 + 8 * kp);
                const int a0 = d0.x, na = d0.y;
                const int ab = kp * C::apk;
                const int ae = min(na, ab + C::apk);
                if (!aborted && t0 < tb && ab < ae) {
                    StageView v;
                    v.codes = st;
                    v.sstride = sstride;
                    if (p.xres) {
                        const unsigned char* rs = smem + p.off_res_s;
                        v.x = smem + p.off_res + a0 * 128;
                        v.sx32 = rs + (2 * a0) * sstride * 4;
                        v.sx64 = rs + (p.K / 32 + a0) * sstride * 4;
                        v.sx128 = rs + (p.K / 32 + p.K / 64 + a0 / 2) * sstride * 4;
                    } else {
                        v.x = st + p.off_x;
                        v.sx32 = st + p.off_sx + C::sx32 * C::mpad * 4;
                        v.sx64 = st + p.off_sx + C::sx64 * C::mpad * 4;
                        v.sx128 = st + p.off_sx + C::sx128 * C::mpad * 4;
                    }
                    v.sc = st + p.off_sc;
                    v.zr = p.zeros ? st + p.off_zr : nullptr;
                    v.tb = tb;
                    v.a0 = a0;
                    v.gfirst = d0.w;
                    v.kin = kg.x;
                    v.grow = kg.y;
                    if constexpr (GIDX) consume_gidx<NT, TPW>(v, p, L, band, t0, ab, ae, st + p.off_gi, acc);
                    else if constexpr (MODE == kModeNvfp4 || MODE == kModeMxfp4)
                        consume_fp4<NT, TPW, MODE>(v, L, t0, ab, ae, p.tscale ? __ldg(p.tscale) : 1.0f, acc);
                    else consume<NT, TPW, BF16, MODE>(v, L, t0, ab, ae, g, acc);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[r.s]);
            }
            combine_sets<NT, TPW>(xchg, set, t0, L, acc);
            // the part that completes its band is the last one: finished after the loop
            if (pe == (band + 1) * p.KU && ps > band * p.KU) continue;
            if (set == 0 && !aborted) flush_part<NT, TPW>(p, band, pe, cta, t0, L, acc);
            zero_acc<NT, TPW>(acc);
        }
        if (u0 > it.b0 * p.KU && u1 >= (it.b0 + 1) * p.KU)
            complete_band<NT, TPW>(p, smem, xchg, s_abort, it.b0, cta, set, t0, L, aborted, acc);
    }
    }
}

}  // namespace w4d
