// w4_prefill.cuh -- compute-bound W4A16 kernel for large M (prefill) on the 5th-generation
// tensor cores (tcgen05, accumulators in tensor memory).
//
// Prefill multiplies many tokens by every weight and is limited by tensor-core
// throughput (edgesiliconlab.com article on AWQ vs GPTQ, "The Mathematics of Memory
// Bandwidth Saturation"); weights are unpacked with AND/OR bit tricks right before the
// tensor cores and the next tiles are staged while the current ones are multiplied
// ("Kernel Execution: Marlin vs. ExLlamaV2 INT4 GEMM Micro-Architecture", items 1-3).
//
// Persistent CTAs (one per SM) walk tiles of 128 output rows x 256 tokens of
// Y^T = What * X'^T (CTA t takes tiles t, t + gridDim.x, ...), 16 warps in four warpgroups:
//   warp 0      TMA: activation tile (2-D tensor map, 128B swizzle) + packed weight tiles
//               of one 128-row band (1-D bulk copy) + zero-point rows into a 4-slot load
//               ring;
//   warp 1      allocates tensor memory and issues tcgen05.mma (one elected lane): A = the
//               dequantised weights (K-major, 128B swizzle, shared memory), B = the
//               activations, D = fp32 in tensor memory; one 128 x 256 x 16 MMA per 16-deep
//               step;
//   warps 2-7   unpack the packed tiles into exact integers q - z (fp16/bf16) in the
//               swizzled A layout, into a 2-slot ring of their own (the load ring runs
//               further ahead than the dequantised tiles need to);
//   warps 8-15  epilogue: after each quantisation group the MMA warp hands over that
//               group's fp32 partial tile (two tensor-memory buffers, ping-pong); each
//               thread owns one output row and one 128-token half, multiplies the partial
//               by the row's group scale and adds it to register accumulators; at the
//               tile's end it stores Y through a staging buffer.
// Each dequantised 128 x 64 tile serves 256 tokens: per MAC the dequant work and the
// shared-memory traffic (operand reads plus the dequantised and TMA writes) are lower
// than with 256 rows x 128 tokens, which the earlier tiling used.
// With act-order g_idx the scale is folded into fp16 weights instead and the whole K
// accumulates in one tensor-memory buffer.
#pragma once
#include "w4_common.cuh"
#include "w4_fp4.cuh"

namespace w4p {

// Weight formats of the prefill kernel.
enum : int {
    kWInt4 = 0,    // INT4 codes, contiguous groups: per-group fp32 rescale of TMEM partials
    kWGidx = 1,    // INT4 codes, act-order g_idx: the scale folded into each fp16 weight
    kWNvfp4 = 2,   // NVFP4: E2M1 x E4M3 block scale, exact in fp16; tensor scale at the end
    kWMxfp4 = 3,   // MXFP4: E2M1 x 2^e, exact in fp16 for e in [-13, 13]
};

constexpr int BN = 128;        // output rows per tile (MMA M)
constexpr int BM = 256;        // tokens per tile (MMA N)
constexpr int BK = 64;         // input channels per stage (one 128-byte swizzle row)
constexpr int kLoadStages = 4;  // activations, codes, zero points: the copies run this far ahead
constexpr int kDeqStages = 2;   // dequantised weight tiles (double-buffered)
constexpr int kThreads = 512;  // producer, MMA, 6 dequant, 8 epilogue warps (4 warpgroups)
constexpr int kDequantWarps = 6;
// Register split: launched with 128 registers a thread (512 x 128 = the SM's 65536);
// warpgroups 0-1 (producer, MMA, dequant) give theirs down to kRegsLow, warpgroups 2-3
// (epilogue: 128 fp32 accumulators plus a 32-column tensor-memory load a thread) take
// kRegsHigh.  2 x 128 x 80 + 2 x 128 x 176 = 65536, exactly the launch's registers; with
// 168 for the epilogue its per-group loop spilled to local memory.
constexpr int kLaunchRegs = 128;
constexpr int kRegsLow = 80;
constexpr int kRegsHigh = 176;
static_assert(2 * 128 * kRegsLow + 2 * 128 * kRegsHigh <= kThreads * kLaunchRegs, "register split");
constexpr int kTmemCols = 512; // two fp32 partial buffers x BM columns
constexpr int kYChunk = 32;    // tokens of each token half per pass of the output staging buffer

constexpr int kABytes = BN * BK * 2;   // 16 KB dequantised operand tile
constexpr int kBBytes = BM * BK * 2;   // 32 KB activation tile
constexpr int kPBytes = BN * BK / 2;   // 4 KB packed codes (one 128-row band)
constexpr int kZBytes = 2 * BN * 2;    // zero-point rows of up to two groups
constexpr int kStageBytes = kABytes + kBBytes + kPBytes + kZBytes;

struct SmemLayout {
    static constexpr int a = 0;                              // kDeqStages x 16 KB (1024-aligned)
    static constexpr int b = a + kDeqStages * kABytes;       // kLoadStages x 32 KB
    static constexpr int pk = b + kLoadStages * kBBytes;     // kLoadStages x 4 KB
    static constexpr int zr = pk + kLoadStages * kPBytes;    // kLoadStages x 512 B
    static constexpr int y = zr + kLoadStages * kZBytes;     // output staging: 2 x kYChunk x BN fp32
    static constexpr int bars = y + 2 * kYChunk * BN * 4;    // barriers
    static constexpr int nbars = 2 * kLoadStages + 2 * kDeqStages + 4 + 1;
    static constexpr int tmem_slot = bars + nbars * 8;
    static constexpr int flags = tmem_slot + 8;
    static constexpr int bytes = flags + 16 + 1024;          // + alignment slack
};

struct PrefillParams {
    const uint32_t* qw;
    const __half* scales;
    const __half* zeros;
    const int32_t* g_idx;
    const uint8_t* bscale;   // FP4 block scales [K/B, N]
    const float* tscale;     // NVFP4 tensor scale (device fp32) or null
    void* Y;
    int M, N, K, group_size, G, out_dtype;
    int KA;       // K / 64
    int tiles;    // N / 16
};

// ---------------------------------------------------------------- tcgen05 wrappers
// d = a * b + d on two fp32 lanes at once (sm_100 packed fp32 FMA; each lane rounds as
// fmaf does).
W4_DEV void fma2(float& d0, float& d1, float a, float b0, float b1) {
    asm("{\n\t.reg .b64 pa, pb, pd;\n\t"
        "mov.b64 pa, {%2, %2};\n\tmov.b64 pb, {%3, %4};\n\tmov.b64 pd, {%0, %1};\n\t"
        "fma.rn.f32x2 pd, pa, pb, pd;\n\tmov.b64 {%0, %1}, pd;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a), "f"(b0), "f"(b1));
}

W4_DEV void tmem_alloc(uint32_t* slot, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                     smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
}
W4_DEV void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
W4_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}
W4_DEV void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
W4_DEV void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

W4_DEV void tc_commit(uint64_t* bar) {
    asm volatile(
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
            smem_u32(bar))
        : "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (fp16 or bf16 in, fp32 out)
W4_DEV void tc_mma(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                   uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// 32 lanes x 32 consecutive fp32 columns: thread i of the warp gets its lane's 32 values.
W4_DEV void tmem_ld32(uint32_t taddr, float (&v)[32]) {
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
          "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
          "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
          "=r"(r[31])
        : "r"(taddr)
        : "memory");
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor: K-major tile whose rows are 128-byte swizzled lines,
// 8-row groups 1024 bytes apart (the layout TMA writes with 128B swizzle).
W4_DEV uint64_t sw128_desc(uint32_t saddr) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);          // start address
    d |= (uint64_t)1u << 16;                           // leading byte offset (unused here)
    d |= (uint64_t)(1024u >> 4) << 32;                 // stride byte offset: 8 rows
    d |= (uint64_t)1u << 46;                           // descriptor version
    d |= (uint64_t)2u << 61;                           // 128-byte swizzle
    return d;
}

// Instruction descriptor: fp32 accumulator, A/B fp16 (0) or bf16 (1), both K-major,
// N = BM tokens, M = BN rows (a single-CTA MMA is at most 128 rows and 256 columns).
W4_DEV uint32_t mma_idesc(bool bf16) {
    const uint32_t fmt = bf16 ? 1u : 0u;
    return (1u << 4) | (fmt << 7) | (fmt << 10) | ((uint32_t)(BM >> 3) << 17) |
           ((uint32_t)(BN >> 4) << 24);
}

// Per-warpgroup register limits (executed by all 128 threads of a warpgroup).  An increase
// waits until the registers are free, so the split must fit the launch's registers; the
// host launches the kernel only when it was compiled with kLaunchRegs registers a thread.
template <uint32_t N>
W4_DEV void setmaxnreg_inc() {
    asm volatile("setmaxnreg.inc.sync.aligned.u32 %0;" ::"n"(N));
}
template <uint32_t N>
W4_DEV void setmaxnreg_dec() {
    asm volatile("setmaxnreg.dec.sync.aligned.u32 %0;" ::"n"(N));
}

// Store four 8x8 16-bit matrices from the MMA fragment layout to shared memory; each
// lane gives the address of one 16-byte row (lanes 8i..8i+7: rows of matrix i).
W4_DEV void stmatrix_x4(uint32_t saddr, const uint32_t (&r)[4]) {
    asm volatile("stmatrix.sync.aligned.m8n8.x4.shared.b16 [%0], {%1, %2, %3, %4};" ::"r"(saddr),
                 "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3])
                 : "memory");
}

W4_DEV void store_out(const PrefillParams& p, int m, int n, float v) {
    const size_t idx = (size_t)m * p.N + n;
    if (p.out_dtype == 2) reinterpret_cast<float*>(p.Y)[idx] = v;
    else if (p.out_dtype == 1) reinterpret_cast<__nv_bfloat16*>(p.Y)[idx] = __float2bfloat16_rn(v);
    else reinterpret_cast<__half*>(p.Y)[idx] = __float2half_rn(v);
}

// bounded wait that also honours the CTA's abort flag (read only when the phase is not
// already complete)
W4_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort_flag) {
    if (mbar_try_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    if (mbar_wait(bar, parity)) return true;
    *abort_flag = 1;
    return false;
}

template <bool BF16, int WM>
__global__ void __launch_bounds__(kThreads, 1)
    prefill_kernel(const __grid_constant__ CUtensorMap tmap_x, const PrefillParams p) {
    constexpr bool GIDX = WM == kWGidx;
    constexpr bool FP4 = WM == kWNvfp4 || WM == kWMxfp4;
    constexpr bool ONEBUF = GIDX || FP4;   // scale in the weights: one partial over the whole K
    extern __shared__ unsigned char smem_raw[];
    // 1024-byte alignment for the swizzled operand tiles
    unsigned char* smem = align_smem_1024(smem_raw);
    using L = SmemLayout;
    uint64_t* full = reinterpret_cast<uint64_t*>(smem + L::bars);
    uint64_t* empty = full + kLoadStages;    // load slot free (its stage's MMAs are done)
    uint64_t* deq = empty + kLoadStages;     // dequantised tile written
    uint64_t* wempty = deq + kDeqStages;     // dequantised tile consumed by the MMAs
    uint64_t* pfull = wempty + kDeqStages;   // [2]
    uint64_t* pempty = pfull + 2;            // [2]
    uint64_t* mma_done = pempty + 2;         // [1]
    uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(smem + L::tmem_slot);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(smem + L::flags);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int KT = p.K / BK;              // stages along K per tile
    const int g = p.group_size;
    const int ngroups = ONEBUF ? 1 : p.K / g;
    // persistent tiles: tile t covers tokens [m0, m0+BM) of m-block t / nbands and output
    // rows [n0, n0+BN) of row block t % nbands, so the CTAs running at one time share
    // their activation tiles (L2 reuse); a CTA takes tiles blockIdx.x, + gridDim.x, ...
    const int nbands = (p.N + BN - 1) / BN;
    const int ntiles = nbands * ((p.M + BM - 1) / BM);

    if (threadIdx.x == 0) {
        for (int s = 0; s < kLoadStages; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int s = 0; s < kDeqStages; ++s) {
            mbar_init(&deq[s], 32 * kDequantWarps);
            mbar_init(&wempty[s], 1);
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&pfull[b], 1);
            mbar_init(&pempty[b], 256);
        }
        mbar_init(mma_done, 1);
        *abort_flag = 0;
        fence_mbar_init();
    }
    if (warp == 1) {
        tmem_alloc(tmem_slot, kTmemCols);
        tmem_relinquish();
    }
    if (warp == 0 && lane == 0) prefetch_tensormap(&tmap_x);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_slot;
    // The next kernel may be scheduled while this grid runs; codes and zero points, read
    // before pdl_wait(), are never written by the kernels of this library.
    pdl_launch_dependents();
    if (warp < 8) {
    // warpgroups 0-1: producer, MMA issuer, dequant warps (few registers each)
    setmaxnreg_dec<kRegsLow>();
    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            // the codes of one 128-row band for column block kt are one contiguous run of
            // tiles x 512 bytes; a tile of BN rows spans two bands
            int gst = 0;   // stage counter across this CTA's tiles (ring slot, phase)
            bool waited = false;
            for (int t = blockIdx.x; t < ntiles && !*abort_flag; t += gridDim.x) {
                const int rb = t % nbands;
                const int n0 = rb * BN, m0 = (t / nbands) * BM;
                const int th = max(0, min(BN / 16, p.tiles - n0 / 16));   // 16-row tiles
                const int zgroups = (!ONEBUF && p.zeros) ? (g == 32 ? 2 : 1) : 0;
                const uint32_t bytes = kBBytes + th * (512 + zgroups * 32);
                for (int kt = 0; kt < KT; ++kt, ++gst) {
                    const int s = gst % kLoadStages, ph = (gst / kLoadStages) & 1;
                    if (gst >= kLoadStages && !wait_or_abort(&empty[s], ph ^ 1, abort_flag)) break;
                    mbar_arrive_expect_tx(&full[s], bytes);
                    bulk_g2s(smem + L::pk + s * kPBytes, p.qw + 128 * ((size_t)8 * p.KA * rb + (size_t)kt * th),
                             th * 512, &full[s]);
                    for (int zg = 0; zg < zgroups; ++zg)
                        bulk_g2s(smem + L::zr + s * kZBytes + zg * BN * 2,
                                 p.zeros + (size_t)((kt * BK) / g + zg) * p.N + n0, th * 32, &full[s]);
                    if (!waited) {
                        pdl_wait();   // activations may come from the preceding kernel
                        waited = true;
                    }
                    tma_load_2d(smem + L::b + s * kBBytes, &tmap_x, kt * BK, m0, &full[s]);
                }
            }
            if (*abort_flag)
                for (int i = (gst > kLoadStages ? gst - kLoadStages : 0); i < gst; ++i)
                    (void)mbar_wait(&full[i % kLoadStages], (i / kLoadStages) & 1);
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        // the whole warp runs the loop (its values stay warp-uniform); one elected lane
        // issues each MMA and commit.  Per 16-channel step: one 128x256x16 MMA.
        const bool leader = elect_one();
        const uint32_t idesc = mma_idesc(BF16 && !GIDX);
        // descriptors of slot 0 of each ring; slot s and 16-channel step j are
        // s * (tile bytes) + 32 j bytes further (>> 4 in the descriptors)
        const uint64_t a_desc0 = sw128_desc(smem_u32(smem + L::a));
        const uint64_t b_desc0 = sw128_desc(smem_u32(smem + L::b));
        // group boundaries: every spg stages (g a multiple of 64), twice per stage
        // (g = 32) or once per tile (act-order: one partial sum over the whole K)
        const int spg = ONEBUF ? KT : (g >= BK ? g / BK : 1);
        const bool two_per_stage = !ONEBUF && g == 32;
        int grp_i = -1;   // group counter across this CTA's tiles (partial buffer, phase)
        int gst = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            int sig = 0;   // stage index inside the current group
            for (int kt = 0; kt < KT; ++kt, ++gst) {
                const int s = gst % kLoadStages, ds = gst % kDeqStages;
                const uint32_t ph = (uint32_t)((gst / kDeqStages) & 1);
                // the dequant warps arrive on deq[ds] only after full[s] completed (the
                // activation tile landed), so deq[ds] alone orders the MMA after both
                ok = wait_or_abort(&deq[ds], ph, abort_flag);
                if (!__all_sync(0xffffffffu, ok)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                const uint64_t ad = a_desc0 + (uint64_t)(ds * (kABytes >> 4));
                const uint64_t bd = b_desc0 + (uint64_t)(s * (kBBytes >> 4));
#pragma unroll
                for (int hk = 0; hk < 2; ++hk) {
                    // hk: 32-channel half of the stage
                    const bool starts = two_per_stage ? true : (hk == 0 && sig == 0);
                    if (starts) {
                        ++grp_i;
                        if (grp_i >= 2) {
                            ok = wait_or_abort(&pempty[grp_i & 1], ((grp_i >> 1) - 1) & 1, abort_flag);
                            ok = __all_sync(0xffffffffu, ok);
                            if (!ok) break;
                            tc_fence_after();
                        }
                    }
                    const uint32_t dcol = tmem_base + (uint32_t)((grp_i & 1) * BM);
                    if (leader) {
#pragma unroll
                        for (int j = 0; j < 2; ++j)
                            tc_mma(dcol, ad + 4 * hk + 2 * j, bd + 4 * hk + 2 * j, idesc,
                                   (starts && j == 0) ? 0u : 1u);
                    }
                    const bool ends = two_per_stage ? true : (hk == 1 && sig == spg - 1);
                    if (ends && leader) tc_commit(&pfull[grp_i & 1]);
                }
                if (!ok) break;
                if (leader) {
                    tc_commit(&empty[s]);      // the load slot (activations) is free
                    tc_commit(&wempty[ds]);    // and so is the dequantised tile
                }
                if (++sig == spg) sig = 0;
            }
        }
        // every MMA this warp issued has finished once mma_done completes
        if (leader) tc_commit(mma_done);
        (void)mbar_wait(mma_done, 0);
        __syncwarp();
    } else if (warp < 8) {
        // ------------------------------------------------------------ dequant warps
        const int dq = warp - 2;                 // row tiles dq and dq + 6 of the 8
        const int gq = lane >> 2, c = 2 * (lane & 3);
        // stmatrix.x4 row addresses: lane l gives row (l & 7) of 8x8 matrix l >> 3, the
        // matrices being (rows 0-7 | 8-15) x (channels 0-7 | 8-15) of a 16x16 step, i.e.
        // the order of the MMA A fragment the unpack produces
        const int mi = lane >> 3, rr = lane & 7;
        int gst = 0;
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles && ok; t += gridDim.x) {
            const int n0 = (t % nbands) * BN;
            const int tt_end = max(0, min(BN / 16, p.tiles - n0 / 16));   // tiles of the tile
            for (int kt = 0; kt < KT; ++kt, ++gst) {
                const int s = gst % kLoadStages, ph = (gst / kLoadStages) & 1;
                const int ds = gst % kDeqStages, dph = (gst / kDeqStages) & 1;
                // the stage's copies have landed and the MMAs are done with the tile slot
                if (!wait_or_abort(&full[s], ph, abort_flag) ||
                    (gst >= kDeqStages && !wait_or_abort(&wempty[ds], dph ^ 1, abort_flag))) {
                    ok = false;
                    break;
                }
#pragma unroll 1
                for (int ti = dq; ti < BN / 16; ti += kDequantWarps) {
                    if (ti >= tt_end) break;
                    const int tt = ti;
                    const uint32_t a_u32 = smem_u32(smem + L::a + ds * kABytes);
                    const unsigned char* pk = smem + L::pk + s * kPBytes;
                    const unsigned char* zs = smem + L::zr + s * kZBytes;
                    const uint4 wq = *reinterpret_cast<const uint4*>(pk + tt * 512 + lane * 16);
                    const uint32_t wv[4] = {wq.x, wq.y, wq.z, wq.w};
                    const int r0 = 16 * tt + gq, r1 = r0 + 8;      // rows within the tile
                    const int nr0 = n0 + r0, nr1 = nr0 + 8;            // output rows
                    const uint32_t row_addr = a_u32 + (uint32_t)((16 * tt + rr + 8 * (mi & 1)) * 128);
                    // zero-point constants of this stage's group(s) (two groups when g = 32)
                    ZeroConsts zc[2];
                    if constexpr (!ONEBUF) {
#pragma unroll
                        for (int zg = 0; zg < 2; ++zg) {
                            const int zo = (g == 32 ? zg : 0) * BN * 2;
                            const uint32_t z0 = p.zeros ? *reinterpret_cast<const unsigned short*>(zs + zo + 2 * r0) : 0x4800u;
                            const uint32_t z1 = p.zeros ? *reinterpret_cast<const unsigned short*>(zs + zo + 2 * r1) : 0x4800u;
                            zc[zg] = zero_consts_h<BF16>(z0, z1);
                        }
                    }
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        const int kk = 16 * j + c;                 // column within the stage
                        const int kabs = kt * BK + kk;
                        uint32_t af[4];
                        if constexpr (FP4) {
                            // E2M1 (exact fp16) times the block's scale (exact fp16 product)
                            constexpr int B = WM == kWNvfp4 ? 16 : 32;
                            const int blk = (kt * BK + 16 * j) / B;
                            const uint32_t b0 = __ldg(p.bscale + (size_t)blk * p.N + nr0);
                            const uint32_t b1 = __ldg(p.bscale + (size_t)blk * p.N + nr1);
                            uint32_t s0, s1;
                            if constexpr (WM == kWNvfp4) {
                                s0 = w4f::e4m3x2_to_h2(b0 | (b0 << 8));
                                s1 = w4f::e4m3x2_to_h2(b1 | (b1 << 8));
                            } else {
                                // 2^(b-127) as fp16; blocks outside [-13, 13] (other than the
                                // all-but-zero byte 0) cannot be decoded exactly: reported
                                const int e0 = (int)b0 - 127, e1 = (int)b1 - 127;
                                if ((b0 != 0 && (e0 < -13 || e0 > 13)) || (b1 != 0 && (e1 < -13 || e1 > 13)))
                                    atomicOr(&g_w4_error_word, W4_DEVERR_GIDX);
                                const uint32_t h0 = (e0 < -14 || e0 > 15) ? 0u : (uint32_t)(e0 + 15) << 10;
                                const uint32_t h1 = (e1 < -14 || e1 > 15) ? 0u : (uint32_t)(e1 + 15) << 10;
                                s0 = h0 | (h0 << 16);
                                s1 = h1 | (h1 << 16);
                            }
                            w4f::unpack_fp4(wv[j], af);
                            af[0] = h2_as_u32(__hmul2(u32_as_h2(af[0]), u32_as_h2(s0)));
                            af[1] = h2_as_u32(__hmul2(u32_as_h2(af[1]), u32_as_h2(s1)));
                            af[2] = h2_as_u32(__hmul2(u32_as_h2(af[2]), u32_as_h2(s0)));
                            af[3] = h2_as_u32(__hmul2(u32_as_h2(af[3]), u32_as_h2(s1)));
                        } else if constexpr (!GIDX) {
                            unpack_word<BF16>(wv[j], zc[j >> 1], af);
                        } else {
                            int gk[4] = {__ldg(p.g_idx + kabs), __ldg(p.g_idx + kabs + 1),
                                         __ldg(p.g_idx + kabs + 8), __ldg(p.g_idx + kabs + 9)};
#pragma unroll
                            for (int e = 0; e < 4; ++e)
                                if (gk[e] < 0 || gk[e] >= p.G) {
                                    atomicOr(&g_w4_error_word, W4_DEVERR_GIDX);
                                    gk[e] = 0;
                                }
#pragma unroll
                            for (int r = 0; r < 4; ++r) {
                                const int row = (r & 1) ? nr1 : nr0;
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
                        }
                        // 128B-swizzled K-major rows: chunk (2j + mi/2) of row r at (chunk ^ (r & 7))
                        stmatrix_x4(row_addr + (uint32_t)((((2 * j + (mi >> 1)) ^ rr) & 7) << 4), af);
                    }
                }
                fence_proxy_async_smem();
                mbar_arrive(&deq[ds]);
            }
        }
    }
    } else {
        // ------------------------------------------------------------ epilogue warps
        // warpgroups 2-3: 128 fp32 accumulators a thread
        setmaxnreg_inc<kRegsHigh>();
        pdl_wait();   // before any store to Y
        const int e = warp - 8;
        const int quad = warp & 3;                 // tensor-memory lanes 32*quad..
        const int h = e >> 2;                      // token half: columns 128 h ..
        const int row = 32 * quad + lane;          // output row within the tile
        const int esz = p.out_dtype == 2 ? 4 : 2;
        unsigned char* yt = smem + L::y;
        int ge = 0;   // group counter across this CTA's tiles (partial buffer, phase)
        bool ok = true;
        for (int t = blockIdx.x; t < ntiles; t += gridDim.x) {
            const int n0 = (t % nbands) * BN, m0 = (t / nbands) * BM;
            const int n = n0 + row;
            const bool row_ok = n < p.N;
            float acc[BM / 2];
#pragma unroll
            for (int i = 0; i < BM / 2; ++i) acc[i] = 0.0f;
            for (int grp = 0; grp < ngroups && ok; ++grp, ++ge) {
                const int pb = ge & 1;
                float sc = 1.0f;
                if constexpr (FP4) sc = p.tscale ? __ldg(p.tscale) : 1.0f;
                else if (!GIDX && row_ok) sc = __half2float(__ldg(p.scales + (size_t)grp * p.N + n));
                ok = wait_or_abort(&pfull[pb], (ge >> 1) & 1, abort_flag);
                if (!ok) break;
                tc_fence_after();
                const uint32_t taddr = tmem_base + ((uint32_t)(32 * quad) << 16) + (uint32_t)(pb * BM + h * (BM / 2));
#pragma unroll
                for (int ch = 0; ch < BM / 64; ++ch) {
                    float v[32];
                    tmem_ld32(taddr + 32 * ch, v);
#pragma unroll
                    for (int i = 0; i < 32; i += 2) fma2(acc[32 * ch + i], acc[32 * ch + i + 1], sc, v[i], v[i + 1]);
                }
                tc_fence_before();
                mbar_arrive(&pempty[pb]);
            }
            // Y tile through a staging buffer of kYChunk tokens of each token half: thread
            // `row` of half h writes column `row` of rows h kYChunk .. of a [2 kYChunk
            // tokens][BN rows] block, then the eight warps copy it out in 16-byte pieces
            // along N.  The next tile's MMAs proceed meanwhile.
            const int cpr = BN * esz / 16;               // 16-byte pieces per token row
            const int ncols = min(BN, p.N - n0);         // a multiple of 16 (N % 16 == 0)
#pragma unroll
            for (int ck = 0; ck < BM / 2 / kYChunk; ++ck) {
                if (ok) {
#pragma unroll
                    for (int i = 0; i < kYChunk; ++i) {
                        unsigned char* ep = yt + ((h * kYChunk + i) * BN + row) * esz;
                        const float v = acc[ck * kYChunk + i];
                        if (p.out_dtype == 2) *reinterpret_cast<float*>(ep) = v;
                        else if (p.out_dtype == 1) *reinterpret_cast<__nv_bfloat16*>(ep) = __float2bfloat16_rn(v);
                        else *reinterpret_cast<__half*>(ep) = __float2half_rn(v);
                    }
                }
                named_bar_sync(1, 256);
                if (ok) {
                    for (int cc = 32 * e + lane; cc < 2 * kYChunk * cpr; cc += 256) {
                        const int m = cc / cpr, pc = cc - m * cpr;
                        const int mm = m0 + (m / kYChunk) * (BM / 2) + ck * kYChunk + m % kYChunk;
                        if (mm >= p.M || pc * 16 >= ncols * esz) continue;
                        const uint4 v = *reinterpret_cast<const uint4*>(yt + m * BN * esz + pc * 16);
                        *reinterpret_cast<uint4*>(reinterpret_cast<unsigned char*>(p.Y) +
                                                  ((size_t)mm * p.N + n0) * esz + pc * 16) = v;
                    }
                }
                named_bar_sync(1, 256);   // the buffer is free for the next block
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, kTmemCols);
    }
}

// X'[m,k] = X[m,k] * s_inv[k], rounded to the activation type (for the prefill path,
// whose activations reach the tensor cores straight from TMA).
template <bool BF16>
__global__ void scale_acts_kernel(const void* __restrict__ X, const float* __restrict__ s_inv,
                                  void* __restrict__ Xp, int M, int K) {
    const size_t pairs = (size_t)M * K / 2;
    const uint32_t* xin = reinterpret_cast<const uint32_t*>(X);
    uint32_t* xout = reinterpret_cast<uint32_t*>(Xp);
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < pairs;
         i += (size_t)gridDim.x * blockDim.x) {
        const int k = (int)((2 * i) % K);
        const float2 v = unpack2<BF16>(xin[i]);
        const float2 s = *reinterpret_cast<const float2*>(s_inv + k);
        xout[i] = pack2<BF16>(__fmul_rn(v.x, s.x), __fmul_rn(v.y, s.y));
    }
}

}  // namespace w4p
