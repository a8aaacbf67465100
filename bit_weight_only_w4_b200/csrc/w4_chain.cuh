// w4_chain.cuh -- a sequence of decode GEMMs (M <= 8) in one persistent launch.
//
// A decode step reads every weight once per token and is limited by memory bandwidth
// (edgesiliconlab.com article on AWQ vs GPTQ, "The Mathematics of Memory Bandwidth
// Saturation": tokens/s is bounded by bandwidth over the bytes of the model).  Launched
// one GEMM at a time, every projection pays a fixed head (barrier set-up, activations,
// first copies) and tail (the split-K completion of the last bands) during which HBM
// idles.  Here one grid of one CTA per SM runs a list of layers: the copy warp streams
// the packed weights of layer after layer into the ring without waiting (weights never
// depend on activations), so while the CTAs finish layer l and wait for each other,
// layer l+1's weights are already in flight.
//
// Layer l+1 may read any earlier layer's output.  Between layers every CTA arrives on a
// counter in the workspace once its share of layer l (its stores and published split-K
// partials) is done, and waits (bounded) for all CTAs' arrivals before it prepares
// layer l+1's X' from global memory (read through L2: written in this launch).  All CTAs
// must be resident at once: the grid is one CTA per SM, each CTA holding more than half
// of the SM's shared memory.  The last CTA to arrive after the last layer zeroes the
// counter for the next launch.
//
// Per layer the work is the decode kernel's with one token tile and resident X'
// (w4_decode.cuh): stream-K units of 128 output rows x 128 input channels, two MMA groups
// on alternate stages, the per-group fold, and the deterministic split-K completion.
#pragma once
#include "w4_decode.cuh"

namespace w4c {

constexpr int kMaxLayers = 32;   // layers per launch (the parameters live in kernel space)

struct ChainParams {
    CUtensorMap sc[kMaxLayers];        // scale rows of each layer (2-D boxes, [G,N])
    CUtensorMap zr[kMaxLayers];        // zero-point rows (unused for symmetric layers)
    w4d::DecodeParams L[kMaxLayers];   // per layer; ring geometry fields equal in all
    unsigned int* counter;             // arrivals between layers (zero at launch)
    int n_layers;
};

// Arrive on the grid counter (release: this CTA's prior writes, ordered before by the
// CTA barrier, become visible to whoever acquires the count).
W4_DEV unsigned int grid_arrive(unsigned int* c) {
    __threadfence();
    unsigned int old;
    asm volatile("atom.add.acq_rel.gpu.global.u32 %0, [%1], 1;" : "=r"(old) : "l"(c) : "memory");
    return old;
}

W4_DEV unsigned int grid_count(const unsigned int* c) {
    unsigned int v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(c) : "memory");
    return v;
}

// Wait (bounded) until the counter reaches `target`.  False on timeout.
W4_DEV bool grid_wait(const unsigned int* c, unsigned int target) {
    if (grid_count(c) >= target) return true;
    const uint64_t t0 = globaltimer_ns();
    const uint64_t limit = *(volatile unsigned long long*)&g_w4_wait_limit_ns;
    for (uint32_t it = 1;; ++it) {
        if (grid_count(c) >= target) break;
        if ((it & 15u) == 0u) {
            if (globaltimer_ns() - t0 > limit) {
                atomicOr(&g_w4_error_word, W4_DEVERR_TIMEOUT);
                return false;
            }
            __nanosleep(32);
        }
    }
    __threadfence();
    return true;
}

template <bool BF16, int MODE>
__global__ void __launch_bounds__(w4d::Cfg<1>::threads, 1)
    chain_kernel(const __grid_constant__ ChainParams cp) {
    using namespace w4d;
    using C = Cfg<1>;
    constexpr int UPS = C::aps / 2;   // units per stage
    const DecodeParams& p0 = cp.L[0];
    const int S = p0.stages;
    const int nl = cp.n_layers;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    unsigned char* xchg = smem + p0.off_xchg;
    uint64_t* full = reinterpret_cast<uint64_t*>(xchg + C::xchg_bytes);
    uint64_t* empty = full + kMaxStages;
    volatile int* s_abort = reinterpret_cast<volatile int*>(empty + kMaxStages);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    constexpr int kConsumers = C::threads - 32;   // activation and MMA warps

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::stage_warps);
        }
        *s_abort = 0;
        fence_mbar_init();
    }
    // activation sums of tokens >= M are never written: start from zero (the region is
    // sized for the largest K of the list)
    {
        const int words = (p0.off_xchg - p0.off_res_s) / 4;
        for (int i = threadIdx.x; i < words; i += C::threads)
            reinterpret_cast<float*>(smem + p0.off_res_s)[i] = 0.0f;
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&cp.sc[0]);
        if (p0.zeros) prefetch_tensormap(&cp.zr[0]);
    }
    __syncthreads();
    // Everything the copy warp reads (codes, scales, zero points) is never written by the
    // kernels of this library, so it runs ahead of pdl_wait() and of the layer barriers.
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------------------ copy warp
        const uint64_t policy = policy_evict_first();
        Ring r;
        int i = 0;
        bool abort = false;
        for (int l = 0; l < nl && !abort; ++l) {
            const DecodeParams& p = cp.L[l];
            const int u0 = unit_begin(p, cta), u1 = unit_begin(p, cta + 1);
            if (u0 >= u1) continue;
            const PartIter it(p, u0, u1);
            const int g = p.group_size;
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
                    if (lane == 0) {
                        unsigned char* st = smem + r.s * p.stage_bytes;
                        const int g_first = (64 * a0) / g;
                        int kg[8] = {0, 0, 0, 0, 0, 0, 0, 0};
#pragma unroll
                        for (int k = 0; k < C::kparts; ++k) {
                            const int off = 64 * a0 - g_first * g + 64 * C::apk * k;
                            kg[2 * k + 1] = off / g;
                            kg[2 * k] = off - kg[2 * k + 1] * g;
                        }
                        int4* desc = reinterpret_cast<int4*>(st + p.off_desc);
                        desc[0] = make_int4(a0, na, tb, g_first);
                        desc[1] = make_int4(kg[0], kg[1], kg[2], kg[3]);
                        desc[2] = make_int4(kg[4], kg[5], kg[6], kg[7]);
                        const uint32_t bytes = na * tb * 512 + p.ngs * p.srow_bytes * (p.zeros ? 2 : 1);
                        mbar_arrive_expect_tx(&full[r.s], bytes);
                        bulk_g2s_hint(st, p.qw + 128 * ((size_t)kTilesPerBand * p.KA * band + (size_t)a0 * tb),
                                      na * tb * 512, &full[r.s], policy);
                        tma_load_2d(st + p.off_sc, &cp.sc[l], band * kBandRows, g_first, &full[r.s]);
                        if (p.zeros) tma_load_2d(st + p.off_zr, &cp.zr[l], band * kBandRows, g_first, &full[r.s]);
                    }
                }
            }
        }
        // On abort, wait (bounded) for the copies already issued before leaving.
        if (abort && lane == 0) {
            Ring q;
            for (int k = 0; k < i; ++k, q.next(S))
                if (k >= i - S) (void)mbar_wait(&full[q.s], q.ph);
        }
        __syncwarp();
        return;
    }

    // ---------------------------------------------------------------- activation and MMA warps
    constexpr int TPW = C::tpw;
    const bool mma = warp > C::xw;
    const int cw = warp - 1 - C::xw;
    const int grp = cw / C::stage_warps, ws = cw % C::stage_warps;
    const int kp = ws / C::tsets;                  // K slice of the stage
    const int t0 = TPW * (ws % C::tsets);          // first row tile
    const int set = grp * C::kparts + kp;          // partial-sum set at a flush
    float acc[TPW][1][4];
    bool aborted = false;
    Ring r;
    int i = 0;
    for (int l = 0; l < nl; ++l) {
        const DecodeParams& p = cp.L[l];
        if (l == 0) {
            pdl_wait();   // X of the first layer may come from the preceding kernel
        } else {
            // this CTA's share of layer l-1 is stored; then every CTA's is
            named_bar_sync(3, kConsumers);
            if (threadIdx.x == 32) {
                grid_arrive(cp.counter);
                if (!grid_wait(cp.counter, gridDim.x * (unsigned)l)) *s_abort = 1;
            }
            named_bar_sync(3, kConsumers);
        }
        int ca0, ca1, cb0, cb1;
        prep_ranges(p, unit_begin(p, cta), unit_begin(p, cta + 1), ca0, ca1, cb0, cb1);
        prep_resident<BF16, false, true>(p, p.X, smem + p.off_res, reinterpret_cast<float*>(smem + p.off_res_s),
                                         warp - 1, C::warps - 1, lane, ca0, ca1, cb0, cb1);
        named_bar_sync(3, kConsumers);
        if (!mma) continue;
        const int u0 = unit_begin(p, cta), u1 = unit_begin(p, cta + 1);
        if (u0 >= u1) continue;
        const PartIter it(p, u0, u1);
        const Lane L = make_lane(lane, p.M, p.sstride, p.K / 64 * 128);
        const int g = p.group_size;
        zero_acc<1, TPW>(acc);
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
                    const unsigned char* rs = smem + p.off_res_s;
                    v.codes = st;
                    v.sstride = p.sstride;
                    v.x = smem + p.off_res + a0 * 128;
                    v.sx32 = rs + (2 * a0) * p.sstride * 4;
                    v.sx64 = rs + (p.K / 32 + a0) * p.sstride * 4;
                    v.sx128 = rs + (p.K / 32 + p.K / 64 + a0 / 2) * p.sstride * 4;
                    v.sc = st + p.off_sc;
                    v.zr = p.zeros ? st + p.off_zr : nullptr;
                    v.tb = tb;
                    v.a0 = a0;
                    v.gfirst = d0.w;
                    v.kin = kg.x;
                    v.grow = kg.y;
                    consume<1, TPW, BF16, MODE>(v, L, t0, ab, ae, g, acc);
                }
                __syncwarp();
                if (lane == 0) mbar_arrive(&empty[r.s]);
            }
            combine_sets<1, TPW>(xchg, set, t0, L, acc);
            if (pe == (band + 1) * p.KU && ps > band * p.KU) continue;   // completed below
            if (set == 0 && !aborted) flush_part<1, TPW>(p, band, pe, cta, t0, L, acc);
            zero_acc<1, TPW>(acc);
        }
        if (u0 > it.b0 * p.KU && u1 >= (it.b0 + 1) * p.KU)
            complete_band<1, TPW>(p, smem, xchg, s_abort, it.b0, cta, set, t0, L, aborted, acc);
    }
    // the last layer is done everywhere once every CTA has arrived; the last arrival
    // zeroes the counter for the next launch (nothing reads it after that)
    named_bar_sync(3, kConsumers);
    if (threadIdx.x == 32) {
        const unsigned int total = gridDim.x * (unsigned)nl;
        if (grid_arrive(cp.counter) == total - 1) atomicExch(cp.counter, 0u);
    }
}

}  // namespace w4c
