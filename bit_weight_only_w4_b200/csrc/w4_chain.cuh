// w4_chain.cuh -- a sequence of decode GEMMs (M <= 8) in one persistent launch.
//
// A decode step reads every weight once per token and is limited by memory bandwidth
// (edgesiliconlab.com article on AWQ vs GPTQ, "The Mathematics of Memory Bandwidth
// Saturation": tokens/s is bounded by bandwidth over the bytes of the model).  Launched
// one GEMM at a time, every projection pays a fixed head (launch, barrier set-up,
// activations, first copies) and tail (the split-K completion of the last bands) during
// which HBM idles.  Here one grid of one CTA per SM runs a list of layers: the copy warp
// streams the packed weights of layer after layer into the ring without waiting (weights
// never depend on activations), so while the CTAs finish layer l and wait for each other,
// layer l+1's weights are already in flight.
//
// Layer l+1 may read any earlier layer's output.  Between layers every CTA arrives on a
// counter in the workspace once its share of layer l (its stores and published split-K
// partials) is done, and waits (bounded) for all CTAs' arrivals before it takes layer
// l+1's X'.  All CTAs must be resident at once: the grid is one CTA per SM, each CTA
// holding more than half of the SM's shared memory.  The last CTA to arrive after the
// last layer zeroes the counter for the next launch.
//
// The layer boundary is on the critical path, so it is kept to a few round trips to L2:
//   - a share warp gathers, while the MMA warps still work, the split-K partials of the
//     band this CTA completes (published by the other contributors) into shared memory,
//     so the completion only adds them;
//   - when X_{l+1} is a 128-aligned column slice of Y_l (the usual chain), the CTA that
//     stores a band of Y_l also writes that band's share of layer l+1's X' (the rounded
//     output times s_inv_{l+1}, in the resident shared-memory image) and of its channel
//     sums (the same sums, in the same order, as the preparation from Y would form) to an
//     exchange buffer; after the barrier one thread of every CTA bulk-copies X' and the
//     sums in, instead of every thread reading Y and s_inv and recomputing them;
//   - the arrival is a release reduction (no round trip waits on it).
//
// Per layer the work is the decode kernel's with one token tile and resident X'
// (w4_decode.cuh): stream-K units of 128 output rows x 128 input channels, two MMA groups
// on alternate stages, the per-group fold, and the deterministic split-K completion (the
// contributors' partials added in CTA order before the completing CTA's own).
#pragma once
#include "w4_decode.cuh"

namespace w4c {

constexpr int kMaxLayers = 32;   // layers per launch (the parameters live in kernel space)
constexpr int kXbufBytes = 120 * 1024;   // one X' exchange buffer: the resident budget
constexpr int kShareFloats = w4d::kTilesPerBand * 4 * 32;   // a band's slot entries, one token tile
constexpr int kWarps = w4d::Cfg<1>::warps + 1;   // copy warp, MMA warps, share warp
constexpr int kThreads = 32 * kWarps;
// shared memory after the exchange buffer: shares [2][kShareFloats] fp32, the next
// layer's s_inv over the completed band [2][128] fp32, the staged outputs of a band
// [8 tokens][128 rows] 16-bit, then the barriers
constexpr int kExtraSmem = 2 * kShareFloats * 4 + 2 * w4d::kBandRows * 4 + 8 * w4d::kBandRows * 2;

struct ChainParams {
    CUtensorMap sc[kMaxLayers];        // scale rows of each layer (2-D boxes, [G,N])
    CUtensorMap zr[kMaxLayers];        // zero-point rows (unused for symmetric layers)
    w4d::DecodeParams L[kMaxLayers];   // per layer; ring geometry fields equal in all
    unsigned int* counter;             // arrivals between layers (zero at launch)
    unsigned char* xbuf[2];            // X' exchange: layer l's X' image, then its sums, in xbuf[l & 1]
    int feed[kMaxLayers];              // 1: layer l's stores also write layer l+1's X'
    int col0[kMaxLayers];              // then X_{l+1} column 0 is column col0[l] of Y_l
    int n_layers;
};

// Arrive on the grid counter: a release reduction, ordered after this CTA's earlier
// writes (which the CTA barrier before it orders before this thread).
W4_DEV void grid_arrive(unsigned int* c) {
    asm volatile("red.release.gpu.global.add.u32 [%0], 1;" ::"l"(c) : "memory");
}

// The last arrival of a launch: returns the count before this one.
W4_DEV unsigned int grid_arrive_last(unsigned int* c) {
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
    return true;
}

// Byte offset of the channel sums in an exchange buffer (after the X' image).
W4_DEV int xbuf_sums_offset(const w4d::DecodeParams& p) { return (p.M * p.K * 2 + 127) / 128 * 128; }

// Store a finished band of layer l (set-0 MMA threads, tid128 = 0..127; every one of
// them calls this, skip or not, since it holds barriers): Y, and when layer l feeds layer
// l+1 and the band is part of X_{l+1}, the band's 128 channels of X'_{l+1} and their
// sums over 32, 64 and 128 channels, written to the exchange buffer exactly as the
// resident preparation of layer l+1 would form them from the stored Y.
// sinv: the next layer's s_inv from the band's first channel on (global memory, or the
// copy the share warp made in shared memory), unused without s_inv.
template <bool BF16, int TPW>
W4_DEV void store_band(const ChainParams& cp, int l, const w4d::DecodeParams& p, int band, int t0,
                       const w4d::Lane& L, const float (&acc)[TPW][1][4], unsigned char* ystage, int tid128,
                       bool skip, const float* sinv) {
    using namespace w4d;
    if (!skip) store_rows<1, TPW>(p, band, t0, L, acc);
    if (!cp.feed[l]) return;
    const DecodeParams& pn = cp.L[l + 1];
    const int k0 = band * kBandRows - cp.col0[l];
    if (k0 < 0 || k0 >= pn.K) return;   // the same for every caller
    unsigned short* ys = reinterpret_cast<unsigned short*>(ystage);
    if (!skip) {
#pragma unroll
        for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                const int m = 2 * L.q + (e & 1);
                if (m < p.M) {
                    const float v = acc[tt][0][e];
                    const uint32_t h = pack2<BF16>(v, v) & 0xFFFFu;
                    ys[m * kBandRows + 16 * (t0 + tt) + L.g8 + 8 * (e >> 1)] = (unsigned short)h;
                }
            }
    }
    named_bar_sync(4, 128);
    const int m = tid128 >> 4, c = tid128 & 15;
    const int k = k0 + 8 * c;
    float s = 0.0f;
    const bool mine = !skip && m < p.M;
    if (mine) {
        uint4 v4 = *reinterpret_cast<const uint4*>(ys + m * kBandRows + 8 * c);
        uint32_t wv[4] = {v4.x, v4.y, v4.z, v4.w};
        if (pn.s_inv) {
            const float4 s0 = reinterpret_cast<const float4*>(sinv + 8 * c)[0];
            const float4 s1 = reinterpret_cast<const float4*>(sinv + 8 * c)[1];
            const float sv[8] = {s0.x, s0.y, s0.z, s0.w, s1.x, s1.y, s1.z, s1.w};
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const float2 f = unpack2<BF16>(wv[i]);
                wv[i] = pack2<BF16>(__fmul_rn(f.x, sv[2 * i]), __fmul_rn(f.y, sv[2 * i + 1]));
            }
        }
        unsigned char* xb = cp.xbuf[(l + 1) & 1];
        *reinterpret_cast<uint4*>(xb + m * (pn.K / 64 * 128) + (k / 64) * 128 + ((((k / 8) & 7) ^ (m & 7)) << 4)) =
            make_uint4(wv[0], wv[1], wv[2], wv[3]);
        float2 f[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) f[i] = unpack2<BF16>(wv[i]);
        s = ((f[0].x + f[0].y) + (f[1].x + f[1].y)) + ((f[2].x + f[2].y) + (f[3].x + f[3].y));
    }
    float* sums = reinterpret_cast<float*>(cp.xbuf[(l + 1) & 1] + xbuf_sums_offset(pn));
    const int ss = pn.sstride;
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (mine && (c & 3) == 0) sums[(k / 32) * ss + m] = s;
    s += __shfl_xor_sync(0xffffffffu, s, 4);
    if (mine && (c & 7) == 0) sums[(pn.K / 32 + k / 64) * ss + m] = s;
    s += __shfl_xor_sync(0xffffffffu, s, 8);
    if (mine && c == 0) sums[(pn.K / 32 + pn.K / 64 + k / 128) * ss + m] = s;
    fence_proxy_async_global();   // other CTAs read the buffer with bulk copies
    named_bar_sync(4, 128);   // the staging tile is free again
}

// Whether CTA `cta` completes a band of layer p: its unit range starts inside a band and
// runs to that band's end.
W4_DEV bool completes_band(const w4d::DecodeParams& p, int cta) {
    const int u0 = w4d::unit_begin(p, cta), u1 = w4d::unit_begin(p, cta + 1);
    if (u0 >= u1) return false;
    const int b0 = u0 / p.KU;
    return u0 > b0 * p.KU && u1 >= (b0 + 1) * p.KU;
}

template <bool BF16, int MODE>
__global__ void __launch_bounds__(kThreads, 1) chain_kernel(const __grid_constant__ ChainParams cp) {
    using namespace w4d;
    using C = Cfg<1>;
    constexpr int UPS = C::aps / 2;   // units per stage
    constexpr int kSlot = kTilesPerBand * 4 * 32;
    const DecodeParams& p0 = cp.L[0];
    const int S = p0.stages;
    const int nl = cp.n_layers;
    extern __shared__ unsigned char smem_raw[];
    unsigned char* smem = align_smem_1024(smem_raw);
    unsigned char* xchg = smem + p0.off_xchg;
    float* shbuf = reinterpret_cast<float*>(xchg + C::xchg_bytes);
    float* sinv_s = shbuf + 2 * kShareFloats;   // [2][128]
    unsigned char* ystage = reinterpret_cast<unsigned char*>(sinv_s + 2 * kBandRows);
    uint64_t* full = reinterpret_cast<uint64_t*>(ystage + 8 * kBandRows * 2);
    uint64_t* empty = full + kMaxStages;
    uint64_t* shbar = empty + kMaxStages;   // [2]: the share warp has gathered a layer's shares
    uint64_t* xbar = shbar + 2;             // the exchange buffer's X' and sums have landed
    volatile int* s_abort = reinterpret_cast<volatile int*>(xbar + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int cta = blockIdx.x;
    constexpr int kConsumers = C::threads - 32;   // the MMA warps
    constexpr int kShareWarp = C::warps;

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], C::stage_warps);
        }
        mbar_init(&shbar[0], 1);
        mbar_init(&shbar[1], 1);
        mbar_init(xbar, 1);
        *s_abort = 0;
        fence_mbar_init();
    }
    // activation sums of tokens >= M are never written by the resident preparation: start
    // from zero (the region is sized for the largest K of the list)
    {
        const int words = (p0.off_xchg - p0.off_res_s) / 4;
        for (int i = threadIdx.x; i < words; i += kThreads)
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

    if (warp == kShareWarp) {
        // ------------------------------------------------------------ share warp
        // For each layer in which this CTA completes a band: the other contributors'
        // partials of that band, summed in CTA order per entry (as the completion of the
        // single-GEMM kernel sums them), into shbuf[l & 1]; then one arrival on shbar[l & 1].
        // The slots of layer l are read only once every CTA has passed into layer l (the
        // grid counter, which only grows within a launch, has every arrival of boundary
        // l): before that a contributor's slot may still hold its layer l-1 partial, which
        // its own completer has yet to take.  By then every CTA is done with layer l-1, so
        // the buffer's previous user, layer l-2, is done with it too.  (An mbarrier phase
        // would not do: this warp can be more than one boundary behind or ahead of the
        // MMA warps, and a parity wait cannot tell such phases apart.)
        pdl_wait();   // the slots may still be in use by the preceding kernel
        for (int l = 0; l < nl; ++l) {
            const DecodeParams& p = cp.L[l];
            const int u0 = unit_begin(p, cta), u1 = unit_begin(p, cta + 1);
            if (u0 >= u1) continue;
            if (!completes_band(p, cta)) continue;
            // `ok` stays the same in every lane (the warp-wide operations below need that)
            bool ok = __shfl_sync(0xffffffffu, *s_abort ? 0 : 1, 0) != 0;
            if (l > 0) {
                // one lane polls (the counter is the layer barrier's hot word)
                int w = 1;
                if (lane == 0) w = (ok && grid_wait(cp.counter, gridDim.x * (unsigned)l)) ? 1 : 0;
                ok = __shfl_sync(0xffffffffu, w, 0) != 0;
            }
            const PartIter it(p, u0, u1);
            float* sh = shbuf + (l & 1) * kShareFloats;
            const int band = it.b0;
            const int c_first = cta_of_unit(p, band * p.KU);
            const int n_ent = band_tiles(p, band) * 16 * p.M;
            // the next layer's s_inv over this band's channels, for the X' the completion
            // writes (in range exactly when the completion writes X')
            if (cp.feed[l] && cp.L[l + 1].s_inv) {
                const int k0 = band * kBandRows - cp.col0[l];
                if (k0 >= 0 && k0 < cp.L[l + 1].K)
                    reinterpret_cast<float4*>(sinv_s + (l & 1) * kBandRows)[lane] =
                        __ldg(reinterpret_cast<const float4*>(cp.L[l + 1].s_inv + k0) + lane);
            }
            // The contributors' entries, up to 2 entries x 8 contributors a lane in flight:
            // rounds of loads of the entries not yet published until all are, then the sums
            // in CTA order and the slots cleared.
            constexpr int E = 2, CB = 8;
            for (int c0 = c_first; c0 < cta && ok; c0 += CB) {
                const int nc = min(CB, cta - c0);
                bool lok = true;
                for (int x0 = lane; x0 < n_ent && lok; x0 += 32 * E) {
                    int j[E];
                    unsigned long long v[E][CB];
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        const int x = x0 + 32 * e;
                        j[e] = x < n_ent ? share_slot<1>(x, p.M) : -1;
#pragma unroll
                        for (int b = 0; b < CB; ++b) v[e][b] = 0ull;
                    }
                    const uint64_t t_start = globaltimer_ns();
                    const uint64_t limit = *(volatile unsigned long long*)&g_w4_wait_limit_ns;
                    for (uint32_t it2 = 0;; ++it2) {
#pragma unroll
                        for (int e = 0; e < E; ++e)
#pragma unroll
                            for (int b = 0; b < CB; ++b)
                                if (j[e] >= 0 && b < nc && (v[e][b] >> 32) == 0)
                                    v[e][b] = slot_get(p.slots + (size_t)(c0 + b) * kSlot + j[e]);
                        bool missing = false;
#pragma unroll
                        for (int e = 0; e < E; ++e)
#pragma unroll
                            for (int b = 0; b < CB; ++b)
                                missing |= j[e] >= 0 && b < nc && (v[e][b] >> 32) == 0;
                        if (!missing) break;
                        if ((it2 & 7u) == 7u && globaltimer_ns() - t_start > limit) {
                            atomicOr(&g_w4_error_word, W4_DEVERR_TIMEOUT);
                            lok = false;
                            break;
                        }
                        __nanosleep(64);
                    }
                    if (!lok) break;
#pragma unroll
                    for (int e = 0; e < E; ++e) {
                        if (j[e] < 0) continue;
                        float t = c0 == c_first ? 0.0f : sh[j[e]];
#pragma unroll
                        for (int b = 0; b < CB; ++b) {
                            if (b >= nc) continue;
                            t += __uint_as_float((uint32_t)v[e][b]);
                            slot_clear(p.slots + (size_t)(c0 + b) * kSlot + j[e]);
                        }
                        sh[j[e]] = t;
                    }
                }
                ok = __all_sync(0xffffffffu, lok) != 0;
            }
            if (!ok) *s_abort = 1;
            __syncwarp();
            if (lane == 0) mbar_arrive(&shbar[l & 1]);
        }
        return;
    }

    // ---------------------------------------------------------------- MMA warps
    constexpr int TPW = C::tpw;
    const int cw = warp - 1;
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
        const bool prepared = l > 0 && cp.feed[l - 1];
        if (l == 0) {
            pdl_wait();   // X of the first layer may come from the preceding kernel
        } else {
            // this CTA's share of layer l-1 is stored; then every CTA's is.  (The resident
            // X' may next be written by a bulk copy: order this thread's accesses to it
            // before that.)
            if (prepared) fence_proxy_async_smem();
            named_bar_sync(3, kConsumers);
            if (threadIdx.x == 32) {
                grid_arrive(cp.counter);
                bool ok = grid_wait(cp.counter, gridDim.x * (unsigned)l);
                if (!ok) *s_abort = 1;
                if (prepared) {
                    // X' and its sums from the exchange buffer (a timed-out wait still
                    // completes the barrier phase, with whatever the buffer holds)
                    fence_proxy_async_global();
                    const unsigned char* src = cp.xbuf[l & 1];
                    const uint32_t img = (uint32_t)(p.M * p.K * 2);
                    const uint32_t sums = (uint32_t)(((p.K / 32 + p.K / 64 + p.K / 128) * p.sstride * 4 + 15) / 16 * 16);
                    mbar_arrive_expect_tx(xbar, img + sums);
                    bulk_g2s(smem + p.off_res, src, img, xbar);
                    bulk_g2s(smem + p.off_res_s, src + (img + 127) / 128 * 128, sums, xbar);
                }
            }
            if (!prepared) named_bar_sync(3, kConsumers);
        }
        if (prepared) {
            // phase: one per earlier layer that took its X' from the exchange buffer
            uint32_t par = 0;
            for (int q = 1; q < l; ++q) par ^= cp.feed[q - 1] ? 1u : 0u;
            if (!mbar_wait(xbar, par)) *s_abort = 1;
        } else {
            prep_resident<BF16, false, true>(p, p.X, smem + p.off_res, reinterpret_cast<float*>(smem + p.off_res_s),
                                             warp - 1, C::warps - 1, lane);
            named_bar_sync(3, kConsumers);
        }
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
            if (set == 0) {
                if (pe < (band + 1) * p.KU) {
                    if (!aborted) flush_part<1, TPW>(p, band, pe, cta, t0, L, acc);   // publish
                } else {
                    const float* sg = cp.feed[l] && cp.L[l + 1].s_inv
                                          ? cp.L[l + 1].s_inv + (band * kBandRows - cp.col0[l]) : nullptr;
                    store_band<BF16, TPW>(cp, l, p, band, t0, L, acc, ystage, threadIdx.x - 32, aborted, sg);
                }
            }
            zero_acc<1, TPW>(acc);
        }
        if (u0 > it.b0 * p.KU && u1 >= (it.b0 + 1) * p.KU) {
            // the band this CTA completes: the share warp's sums of the other
            // contributors' partials, then this CTA's own
            const int b = l & 1;
            if (set == 0) {
                // phase of shbar[b]: one per earlier layer of the same parity that this
                // CTA completed a band of
                uint32_t par = 0;
                for (int q = b; q < l; q += 2) par ^= completes_band(cp.L[q], cta) ? 1u : 0u;
                bool skip = aborted;
                if (!skip && !mbar_wait(&shbar[b], par)) {
                    *s_abort = 1;
                    skip = true;
                }
                skip = skip || *s_abort;
                const int tb = band_tiles(p, it.b0);
                if (!skip) {
                    const float* sh = shbuf + b * kShareFloats;
#pragma unroll
                    for (int tt = 0; tt < TPW; ++tt)
#pragma unroll
                        for (int e = 0; e < 4; ++e)
                            if (t0 + tt < tb && 2 * L.q + (e & 1) < p.M)
                                acc[tt][0][e] = sh[((t0 + tt) * 4 + e) * 32 + lane] + acc[tt][0][e];
                }
                store_band<BF16, TPW>(cp, l, p, it.b0, t0, L, acc, ystage, threadIdx.x - 32, skip,
                                      sinv_s + b * kBandRows);
            }
        }
    }
    // the last layer is done everywhere once every CTA has arrived; the last arrival
    // zeroes the counter for the next launch (nothing reads it after that)
    named_bar_sync(3, kConsumers);
    if (threadIdx.x == 32) {
        const unsigned int total = gridDim.x * (unsigned)nl;
        if (grid_arrive_last(cp.counter) == total - 1) atomicExch(cp.counter, 0u);
    }
}

}  // namespace w4c
