// w4a16.cu -- C ABI of the W4A16 library (declared in include/w4a16.h): argument
// validation, kernel selection by M and launches.  All device work is in the kernels of
// w4_quant.cuh, w4_decode.cuh and w4_prefill.cuh; nothing here touches tensor data.
#include <algorithm>
#include <climits>
#include <cstring>
#include <mutex>

#include "w4a16.h"
#include "w4_common.cuh"
#include "w4_decode.cuh"
#include "w4_prefill.cuh"
#include "w4_quant.cuh"
#include "w4_actorder.cuh"
#include "w4_chain.cuh"
#include "w4_awq.cuh"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kDecodeMaxM = 64;
constexpr int kQuantMaxGroups = 1536;
constexpr int64_t kMaxBands = 8192;                       // N <= 1,048,576 (fix-up counters)
constexpr int64_t kAwqMaxRows = 1 << 19;                  // calibration rows (the reference product's grid.y)

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

cudaStream_t as_stream(w4_stream_t s) { return reinterpret_cast<cudaStream_t>(s); }

w4_status launch_status() {
    return cudaGetLastError() == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

// Shape rules shared by quantisation and GEMM.
w4_status check_layer_shape(int64_t N, int64_t K, int32_t group_size) {
    if (N <= 0 || K <= 0 || group_size <= 0) return W4_ERR_INVALID_ARG;
    if (N > INT_MAX / 2 || K > INT_MAX / 2) return W4_ERR_UNSUPPORTED;
    if (K % group_size != 0) return W4_ERR_INVALID_ARG;
    if (N % 16 != 0 || K % 64 != 0) return W4_ERR_UNSUPPORTED;
    if (N > kMaxBands * 128) return W4_ERR_UNSUPPORTED;
    if (group_size != 32 && group_size % 64 != 0) return W4_ERR_UNSUPPORTED;
    return W4_OK;
}

int current_device() {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess) return -1;
    return dev;
}

int sm_count(int dev) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    return v;
}

// Raise a kernel's dynamic shared-memory limit once per device.
template <typename Kernel>
bool ensure_smem(Kernel k, int bytes, std::once_flag (&flags)[kMaxDevices], int dev) {
    if (bytes <= 48 * 1024) return true;
    if (dev < 0 || dev >= kMaxDevices) return false;
    bool ok = true;
    std::call_once(flags[dev], [&] {
        ok = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) ==
             cudaSuccess;
    });
    // a failure is reported to the first call only; later launches then fail on their own
    return ok;
}

// ---------------------------------------------------------------- decode launch plan
int decode_tiles_for(int64_t M) { return M <= 8 ? 1 : M <= 16 ? 2 : M <= 32 ? 4 : 8; }

// Workspace layout (caller-owned, zero-filled once):
//   [0, 32 KB)                 a fixed region kept at zero (the original counter region;
//                              kept so the layout of the rest is stable);
//   [32 KB, 32 KB + R)         the decode kernel's split-K partial words, one slot of
//                              8 tiles x NT token tiles x 4 x 32 {value, flag} words per CTA
//                              (one CTA per SM).  R is sized for the largest NT (8), so
//                              every decode call -- whatever its M -- finds its slots in the
//                              same place; every call leaves each flag it read at zero;
//   [32 KB + R, ...)           prefill scratch (the activations scaled by s_inv), which
//                              therefore never touches a flag.
constexpr size_t kCounterBytes = (size_t)kMaxBands * 4;   // 32 KB

size_t decode_slot_bytes(int NT, int sms) { return (size_t)sms * w4d::kTilesPerBand * NT * 4 * 32 * 8; }
size_t slot_region_bytes(int sms) { return decode_slot_bytes(8, sms); }

// Behind the zero region and the split-K slots of the largest token-tile count the
// workspace serves (8 for a caller's workspace, whatever the call's M; the no-allocation
// scratch serves at most 4): the decode kernel's prepared activations (X' and its sums;
// prep_acts_kernel), or the prefill kernel's scaled activations.  Calls of different M
// sharing one workspace thus never find another call's activations where their split-K
// flags are.
size_t pre_offset(int max_tiles, int sms) { return kCounterBytes + decode_slot_bytes(max_tiles, sms); }

// Prepared activations of the decode kernel: X' [M, K] (act type), then the sums over 32,
// 64 and 128 channels, [K/32 | K/64 | ceil(K/128)][8 NT] fp32.
struct PreLayout {
    size_t x, s32, s64, s128, bytes;
};
PreLayout pre_layout(int64_t M, int64_t K) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    const size_t mpad = 8 * (size_t)decode_tiles_for(M);
    PreLayout L;
    L.x = 0;
    L.s32 = up((size_t)M * (size_t)K * 2);
    L.s64 = L.s32 + up((size_t)(K / 32) * mpad * 4);
    L.s128 = L.s64 + up((size_t)(K / 64) * mpad * 4);
    L.bytes = L.s128 + up((size_t)((K + 127) / 128) * mpad * 4);
    return L;
}

size_t decode_workspace_bytes(int64_t M, int64_t K, int sms, int max_tiles = 8) {
    return pre_offset(max_tiles, sms) + pre_layout(M, K).bytes;
}

// Act-order GEMM in permuted order with the gather kernel: the gathered activations go
// behind what the GEMM on them uses (the decode kernel prepares its X' from them).
size_t perm_gather_offset(int64_t M, int64_t K, int sms) {
    return M <= kDecodeMaxM ? decode_workspace_bytes(M, K, sms) : pre_offset(8, sms);
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                   const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                   const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_tiled() {
    static EncodeTiledFn fn = [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) !=
                cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            return static_cast<EncodeTiledFn>(nullptr);
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// 2-D map over activations [M,K] (K innermost) with boxes of 64 channels x box_rows rows,
// 128-byte swizzle (the layout the tcgen05 descriptors expect).
bool make_act_tensor_map(CUtensorMap* map, const void* X, bool bf16, int64_t M, int64_t K,
                         int box_rows) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t strides[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {64u, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
               const_cast<void*>(X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D view of prepared activations X' [M,K] as (64 channels, K/64 column blocks, M rows):
// one box of `blocks` column blocks x box_rows rows lands as [row][block][64] (X' is
// stored with its chunks already permuted, so no swizzle here); rows >= M and blocks
// beyond K/64 are zero-filled.
bool make_act_blocks_map(CUtensorMap* map, const void* X, bool bf16, int64_t M, int64_t K,
                         int box_rows, int blocks) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[3] = {64, (cuuint64_t)(K / 64), (cuuint64_t)M};
    const cuuint64_t strides[2] = {128, (cuuint64_t)K * 2};
    const cuuint32_t box[3] = {64u, (cuuint32_t)blocks, (cuuint32_t)box_rows};
    const cuuint32_t estr[3] = {1, 1, 1};
    return enc(map, bf16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 3,
               const_cast<void*>(X), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D map over group metadata [G,N] (N innermost), fp16 or (bytes) uint8: boxes of 128
// columns x rows groups.
bool make_meta_map(CUtensorMap* map, const void* base, int64_t G, int64_t N, int rows, bool bytes = false) {
    EncodeTiledFn enc = encode_tiled();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)N, (cuuint64_t)G};
    const cuuint64_t strides[1] = {(cuuint64_t)N * (bytes ? 1 : 2)};
    const cuuint32_t box[2] = {128u, (cuuint32_t)rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(map, bytes ? CU_TENSOR_MAP_DATA_TYPE_UINT8 : CU_TENSOR_MAP_DATA_TYPE_FLOAT16, 2,
               const_cast<void*>(base), dims, strides,
               box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// X' and its sums stay resident in shared memory (one token tile, M*K small).
bool decode_x_resident(int64_t M, int64_t K) {
    auto up = [](int64_t v, int64_t a) { return (v + a - 1) / a * a; };
    if (M > 8) return false;
    const int64_t sstride = std::max<int64_t>(2, (M + 1) / 2 * 2);
    return up(M * K * 2, 128) + up((K / 32 + K / 64 + K / 128) * sstride * 4, 128) <= 80 * 1024;
}

template <int NT, bool BF16, int MODE, bool PERM>
w4_status launch_decode(w4d::DecodeParams p, const void* X, unsigned char* ws, size_t pre_off, int dev,
                        cudaStream_t stream) {
    using C = w4d::Cfg<NT>;
    constexpr bool GIDX = MODE == w4d::kModeGidx;
    auto kernel = w4d::decode_kernel<NT, BF16, MODE, PERM>;
    static std::once_flag flags[kMaxDevices];
    constexpr int kMaxSmem = 227 * 1024;
    bool attr_ok = true;
    std::call_once(flags[dev], [&] {
        attr_ok = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kMaxSmem) ==
                  cudaSuccess;
    });
    if (!attr_ok) return W4_ERR_CUDA;
    // X' resident (one token tile, small M*K): X' and its sums are prepared once per CTA;
    // the ring then carries only codes and group metadata.
    auto up = [](int v, int a) { return (v + a - 1) / a * a; };
    p.xres = (NT == 1 && !GIDX && decode_x_resident(p.M, p.K)) ? 1 : 0;
    // sizes of the resident X' and sums (decode_x_resident bounds them to 80 KB together)
    const int sstride_res = std::max(2, (int)((p.M + 1) / 2 * 2));
    const int res_x = p.xres ? up(p.M * p.K * 2, 128) : 0;
    const int res_s = p.xres ? up((p.K / 32 + p.K / 64 + p.K / 128) * sstride_res * 4, 128) : 0;
    if (PERM != (p.perm != nullptr) || (PERM && !p.xres))   // the gather is part of the resident X'
        return W4_ERR_UNSUPPORTED;
    p.sstride = p.xres ? sstride_res : C::mpad;
    // stage layout: codes | X' box (8*NT rows) | activation sums | scale rows | zero-point
    // rows | g_idx | descriptor   (no activation parts when X' is resident)
    const int g = p.group_size;
    const int span = 64 * C::aps;   // input channels per stage
    const bool staged_x = !p.xres;
    // FP4: group_size is the scale block (16 or 32), the staged rows are bytes
    constexpr bool FP4 = MODE == w4d::kModeNvfp4 || MODE == w4d::kModeMxfp4;
    p.srow_bytes = FP4 ? 128 : 256;
    p.ngs = GIDX ? 0 : FP4 ? span / g : (g == 32 ? span / 32 : std::min(p.G, (span + 2 * g - 65) / g));
    p.off_x = C::aps * w4d::kTilesPerBand * 512;
    p.off_xs = p.off_x;
    p.off_sx = p.off_x + (staged_x ? C::aps * C::mpad * 128 : 0);
    p.off_si = p.off_sx + (staged_x && !GIDX ? C::sx_floats * 4 : 0);
    p.off_sc = p.off_si;
    p.off_zr = p.off_sc + p.ngs * p.srow_bytes;
    p.off_gi = p.off_zr + (p.zeros ? p.ngs * p.srow_bytes : 0);
    p.off_desc = p.off_gi + (GIDX ? C::aps * 256 : 0);
    p.stage_bytes = (p.off_desc + 48 + 1023) / 1024 * 1024;
    // as many stages as fit: the CTA fills the SM's shared memory, one CTA per SM
    const int resident = p.xres ? res_x + res_s : 0;
    const int fixed = resident + C::xchg_bytes + 3 * w4d::kMaxStages * 8 + 16 + 1024;
    p.stages = std::min(w4d::kMaxStages, (kMaxSmem - fixed) / p.stage_bytes);
    if (p.stages < 2) return W4_ERR_UNSUPPORTED;
    p.off_res = p.stages * p.stage_bytes;
    p.off_res_s = p.off_res + res_x;
    p.off_xchg = p.off_res + resident;
    const int smem = p.stages * p.stage_bytes + fixed;
    p.X = X;
    const int bands = (p.tiles + w4d::kTilesPerBand - 1) / w4d::kTilesPerBand;
    p.KU = (p.KA + 1) / 2;
    p.units = bands * p.KU;
    int P = sm_count(dev);
    if (P <= 0) return W4_ERR_CUDA;
    if (P > p.units) P = p.units;
    p.base = p.units / P;
    p.rem = p.units % P;
    p.slots = reinterpret_cast<unsigned long long*>(ws + kCounterBytes);
    CUtensorMap map_x, map_sc, map_zr;
    std::memset(&map_x, 0, sizeof(map_x));
    if (staged_x) {
        // X' and its sums, prepared once for every CTA (the decode kernel waits for this
        // kernel before it reads them)
        const PreLayout L = pre_layout(p.M, p.K);
        unsigned char* pre = ws + pre_off;
        p.sg32 = reinterpret_cast<const float*>(pre + L.s32);
        p.sg64 = reinterpret_cast<const float*>(pre + L.s64);
        p.sg128 = reinterpret_cast<const float*>(pre + L.s128);
        const size_t threads = (size_t)C::mpad * (size_t)(p.K / 8);
        cudaLaunchConfig_t pc = {};
        pc.gridDim = dim3((unsigned)((threads + 255) / 256));
        pc.blockDim = dim3(256);
        pc.stream = stream;
        cudaLaunchAttribute pa[1];
        pa[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
        pa[0].val.programmaticStreamSerializationAllowed = 1;
        pc.attrs = pa;
        pc.numAttrs = 1;
        if (cudaLaunchKernelEx(&pc, w4d::prep_acts_kernel<BF16>, X, p.s_inv, p.M, p.K, (int)C::mpad,
                               (void*)(pre + L.x), const_cast<float*>(p.sg32), const_cast<float*>(p.sg64),
                               const_cast<float*>(p.sg128)) != cudaSuccess)
            return W4_ERR_CUDA;
        if (!make_act_blocks_map(&map_x, pre + L.x, BF16, p.M, p.K, C::mpad, C::aps)) return W4_ERR_CUDA;
    }
    map_sc = map_x;
    map_zr = map_x;
    if (!GIDX) {
        if (!make_meta_map(&map_sc, p.scales, p.G, p.N, p.ngs, FP4)) return W4_ERR_CUDA;
        if (p.zeros && !make_meta_map(&map_zr, p.zeros, p.G, p.N, p.ngs, FP4)) return W4_ERR_CUDA;
    }
    // programmatic dependent launch: this kernel's prologue and weight loads may overlap
    // the tail of the preceding kernel on the stream
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)P);
    cfg.blockDim = dim3(C::threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, kernel, map_x, map_sc, map_zr, p) != cudaSuccess) return W4_ERR_CUDA;
    return launch_status();
}

// Group handling: one fold per 128-channel half stage when groups are whole multiples of
// 128 channels and K holds whole 128-channel units; a fold per 32 channels for g = 32;
// folds at 64-channel boundaries otherwise.
int decode_mode(int64_t K, int32_t g, bool gidx) {
    if (gidx) return w4d::kModeGidx;
    if (g % 128 == 0 && (K / 64) % 2 == 0) return w4d::kModeHalf;
    if (g == 32) return w4d::kModeG32;
    return w4d::kModeAtom;
}

template <int NT, bool BF16, bool PERM>
w4_status dispatch_mode(int mode, w4d::DecodeParams p, const void* X, unsigned char* ws, size_t pre_off, int dev,
                        cudaStream_t s) {
    if constexpr (!BF16 && !PERM) {
        if (mode == w4d::kModeGidx) return launch_decode<NT, false, w4d::kModeGidx, false>(p, X, ws, pre_off, dev, s);
        if (mode == w4d::kModeNvfp4) return launch_decode<NT, false, w4d::kModeNvfp4, false>(p, X, ws, pre_off, dev, s);
        if (mode == w4d::kModeMxfp4) return launch_decode<NT, false, w4d::kModeMxfp4, false>(p, X, ws, pre_off, dev, s);
    } else {
        if (mode == w4d::kModeGidx || mode == w4d::kModeNvfp4 || mode == w4d::kModeMxfp4) return W4_ERR_UNSUPPORTED;
    }
    if (mode == w4d::kModeHalf) return launch_decode<NT, BF16, w4d::kModeHalf, PERM>(p, X, ws, pre_off, dev, s);
    if (mode == w4d::kModeG32) return launch_decode<NT, BF16, w4d::kModeG32, PERM>(p, X, ws, pre_off, dev, s);
    return launch_decode<NT, BF16, w4d::kModeAtom, PERM>(p, X, ws, pre_off, dev, s);
}

template <bool BF16>
w4_status dispatch_decode(int mode, w4d::DecodeParams p, const void* X, unsigned char* ws, size_t pre_off, int dev,
                          cudaStream_t s) {
    // act-order columns gathered while the resident X' is prepared: one token tile only
    if (p.perm) return decode_tiles_for(p.M) == 1 ? dispatch_mode<1, BF16, true>(mode, p, X, ws, pre_off, dev, s)
                                                  : W4_ERR_UNSUPPORTED;
    switch (decode_tiles_for(p.M)) {
        case 1: return dispatch_mode<1, BF16, false>(mode, p, X, ws, pre_off, dev, s);
        case 2: return dispatch_mode<2, BF16, false>(mode, p, X, ws, pre_off, dev, s);
        case 4: return dispatch_mode<4, BF16, false>(mode, p, X, ws, pre_off, dev, s);
        default: return dispatch_mode<8, BF16, false>(mode, p, X, ws, pre_off, dev, s);
    }
}

// ---------------------------------------------------------------- prefill launch plan
template <bool BF16, int WM>
w4_status launch_prefill(const CUtensorMap& map, const w4p::PrefillParams& p, int dev,
                         cudaStream_t stream) {
    static std::once_flag flags[kMaxDevices];
    auto k = w4p::prefill_kernel<BF16, WM>;
    if (!ensure_smem(k, w4p::SmemLayout::bytes, flags, dev)) return W4_ERR_CUDA;
    // the kernel's per-warpgroup register split assumes this many registers a thread at
    // launch; any other build would make its register increase wait forever
    static int regs[kMaxDevices];
    static std::once_flag rflags[kMaxDevices];
    std::call_once(rflags[dev], [&] {
        cudaFuncAttributes a;
        regs[dev] = cudaFuncGetAttributes(&a, k) == cudaSuccess ? a.numRegs : -1;
    });
    if (regs[dev] != w4p::kLaunchRegs) return W4_ERR_UNSUPPORTED;
    // persistent: one CTA per SM (or per tile when there are fewer tiles)
    const long long ntiles = (long long)((p.N + w4p::BN - 1) / w4p::BN) * ((p.M + w4p::BM - 1) / w4p::BM);
    const int sms = sm_count(dev);
    if (sms <= 0) return W4_ERR_CUDA;
    const dim3 grid((unsigned)std::min<long long>(ntiles, sms));
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(w4p::kThreads);
    cfg.dynamicSmemBytes = (size_t)w4p::SmemLayout::bytes;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k, map, p) != cudaSuccess) return W4_ERR_CUDA;
    return launch_status();
}

}  // namespace

// AWQ scaling + group RTN + packing; with perm (g_idx then NULL) column k of the packed
// matrix is channel perm[k] and groups are contiguous runs of group_size columns.
// Workspace of w4_awq_search: per-channel statistics, the candidate scales, the packed
// candidate, the reference and quantised products, loss partials, the losses, and the
// GEMM's own workspace last (its zero-filled part stays zero between calls).
struct AwqLayout {
    size_t logm, mu, s, s_inv, qw, sc, zr, yref, yq, part, loss, gemm, total;
    int nblk;
};
static AwqLayout awq_layout(int64_t M, int64_t N, int64_t K, int32_t group_size, int32_t symmetric,
                            int32_t n_grid, size_t gemm_bytes) {
    auto up = [](size_t v) { return (v + 255) / 256 * 256; };
    const size_t G = (size_t)(K / group_size);
    const size_t n = (size_t)M * (size_t)N;
    AwqLayout L;
    L.nblk = (int)std::min<size_t>(1024, (n + 4095) / 4096);
    L.logm = 0;
    L.mu = L.logm + up((size_t)K * 8);
    L.s = L.mu + 256;
    L.s_inv = L.s + up((size_t)K * 4);
    L.qw = L.s_inv + up((size_t)K * 4);
    L.sc = L.qw + up((size_t)N * K / 2);
    L.zr = L.sc + up(G * N * 2);
    L.yref = L.zr + (symmetric ? 0 : up(G * N * 2));
    L.yq = L.yref + up(n * 4);
    L.part = L.yq + up(n * 4);
    L.loss = L.part + up((size_t)L.nblk * 8);
    L.gemm = L.loss + up((size_t)n_grid * 8);
    L.total = L.gemm + up(gemm_bytes);
    return L;
}

static w4_status quantize_pack_impl(const void* W, w4_dtype w_dtype, int64_t N, int64_t K, const float* s,
                             int32_t group_size, int32_t symmetric, const int32_t* g_idx,
                             const int32_t* perm, uint32_t* qweight, void* scales, void* zeros,
                             w4_stream_t stream) {
    if (!W || !qweight || !scales) return W4_ERR_INVALID_ARG;
    if (w_dtype != W4_F16 && w_dtype != W4_BF16) return W4_ERR_INVALID_ARG;
    if (symmetric != 0 && symmetric != 1) return W4_ERR_INVALID_ARG;
    if (symmetric ? (zeros != nullptr) : (zeros == nullptr)) return W4_ERR_INVALID_ARG;
    if (!aligned(W, 2) || !aligned(qweight, 4) || !aligned(scales, 2) || !aligned(zeros, 2) ||
        !aligned(s, 4) || !aligned(g_idx, 4) || !aligned(perm, 4))
        return W4_ERR_INVALID_ARG;
    w4_status st = check_layer_shape(N, K, group_size);
    if (st != W4_OK) return st;
    const int64_t G = K / group_size;
    if (G > kQuantMaxGroups) return W4_ERR_UNSUPPORTED;

    w4q::QuantParams p;
    p.W = W;
    p.s = s;
    p.g_idx = g_idx;
    p.perm = perm;
    p.qweight = qweight;
    p.scales = reinterpret_cast<__half*>(scales);
    p.zeros = reinterpret_cast<__half*>(zeros);
    p.N = (int)N;
    p.K = (int)K;
    p.group_size = group_size;
    p.G = (int)G;
    p.symmetric = symmetric;
    const int smem = (int)(2 * w4q::kRows * G * sizeof(int));
    const int dev = current_device();
    if (w_dtype == W4_BF16) {
        static std::once_flag flags[kMaxDevices];
        if (!ensure_smem(w4q::quantize_pack_kernel<true>, 2 * w4q::kRows * kQuantMaxGroups * 4, flags, dev))
            return W4_ERR_CUDA;
        w4q::quantize_pack_kernel<true><<<(unsigned)(N / 16), w4q::kThreads, smem, as_stream(stream)>>>(p);
    } else {
        static std::once_flag flags[kMaxDevices];
        if (!ensure_smem(w4q::quantize_pack_kernel<false>, 2 * w4q::kRows * kQuantMaxGroups * 4, flags, dev))
            return W4_ERR_CUDA;
        w4q::quantize_pack_kernel<false><<<(unsigned)(N / 16), w4q::kThreads, smem, as_stream(stream)>>>(p);
    }
    return launch_status();
}

namespace {
// Zero the allocation-free scratch of device `dev` again if it has been set up (defined
// with the scratch, below).
cudaError_t noalloc_rezero(int dev);
}  // namespace

extern "C" {

const char* w4_status_string(w4_status s) {
    switch (s) {
        case W4_OK: return "W4_OK";
        case W4_ERR_INVALID_ARG: return "W4_ERR_INVALID_ARG";
        case W4_ERR_UNSUPPORTED: return "W4_ERR_UNSUPPORTED";
        case W4_ERR_CUDA: return "W4_ERR_CUDA";
        case W4_ERR_TIMEOUT: return "W4_ERR_TIMEOUT";
        case W4_ERR_DEVICE_ARG: return "W4_ERR_DEVICE_ARG";
    }
    return "W4_ERR_UNKNOWN";
}

w4_status w4_quantize_pack(const void* W, w4_dtype w_dtype, int64_t N, int64_t K, const float* s,
                           int32_t group_size, int32_t symmetric, const int32_t* g_idx,
                           uint32_t* qweight, void* scales, void* zeros, w4_stream_t stream) {
    return quantize_pack_impl(W, w_dtype, N, K, s, group_size, symmetric, g_idx, nullptr, qweight, scales,
                              zeros, stream);
}

w4_status w4_quantize_pack_perm(const void* W, w4_dtype w_dtype, int64_t N, int64_t K, const float* s,
                                int32_t group_size, int32_t symmetric, const int32_t* perm,
                                uint32_t* qweight, void* scales, void* zeros, w4_stream_t stream) {
    if (!perm) return W4_ERR_INVALID_ARG;
    return quantize_pack_impl(W, w_dtype, N, K, s, group_size, symmetric, nullptr, perm, qweight, scales,
                              zeros, stream);
}

w4_status w4_actorder_perm(const int32_t* g_idx, int64_t K, int32_t group_size, int32_t* perm,
                           w4_stream_t stream) {
    if (!g_idx || !perm || !aligned(g_idx, 4) || !aligned(perm, 16)) return W4_ERR_INVALID_ARG;
    if (K <= 0 || K > INT_MAX || group_size <= 0 || K % group_size != 0) return W4_ERR_INVALID_ARG;
    const int64_t G = K / group_size;
    if (G * (int64_t)sizeof(int) > 48 * 1024) return W4_ERR_UNSUPPORTED;
    w4a::actorder_perm_kernel<<<1, 32, (size_t)G * sizeof(int), as_stream(stream)>>>(g_idx, (int)K, group_size,
                                                                                     (int)G, perm);
    return launch_status();
}

size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t group_size) {
    if (M < 0 || check_layer_shape(N, K, group_size) != W4_OK) return 0;
    if (M == 0) return 0;
    const int dev = current_device();
    const int sms = dev >= 0 ? sm_count(dev) : 0;
    if (sms <= 0) return 0;
    if (M <= kDecodeMaxM) return decode_workspace_bytes(M, K, sms);
    // prefill: scaled activations, behind the zero region and the decode slot region
    return kCounterBytes + slot_region_bytes(sms) + (size_t)(((size_t)M * (size_t)K * 2 + 255) / 256 * 256);
}

static w4_status gemm_impl(const void* X, w4_dtype act_dtype, int64_t M, int64_t N, int64_t K,
                           const uint32_t* qweight, const void* scales, const void* zeros,
                           const int32_t* g_idx, const int32_t* perm, int32_t group_size,
                           const float* s_inv, void* Y, w4_dtype out_dtype, void* workspace,
                           size_t workspace_bytes, w4_stream_t stream);

w4_status w4a16_gemm(const void* X, w4_dtype act_dtype, int64_t M, int64_t N, int64_t K,
                     const uint32_t* qweight, const void* scales, const void* zeros,
                     const int32_t* g_idx, int32_t group_size, const float* s_inv, void* Y,
                     w4_dtype out_dtype, void* workspace, size_t workspace_bytes,
                     w4_stream_t stream) {
    return gemm_impl(X, act_dtype, M, N, K, qweight, scales, zeros, g_idx, nullptr, group_size, s_inv, Y,
                     out_dtype, workspace, workspace_bytes, stream);
}

static w4_status gemm_impl(const void* X, w4_dtype act_dtype, int64_t M, int64_t N, int64_t K,
                           const uint32_t* qweight, const void* scales, const void* zeros,
                           const int32_t* g_idx, const int32_t* perm, int32_t group_size,
                           const float* s_inv, void* Y, w4_dtype out_dtype, void* workspace,
                           size_t workspace_bytes, w4_stream_t stream) {
    if (M < 0) return W4_ERR_INVALID_ARG;
    if (act_dtype != W4_F16 && act_dtype != W4_BF16) return W4_ERR_INVALID_ARG;
    if (out_dtype != W4_F16 && out_dtype != W4_BF16 && out_dtype != W4_F32) return W4_ERR_INVALID_ARG;
    w4_status st = check_layer_shape(N, K, group_size);
    if (st != W4_OK) return st;
    if (M == 0) return W4_OK;
    if (M > INT_MAX / 2 || (size_t)M * (size_t)K > (size_t)INT_MAX * 8) return W4_ERR_UNSUPPORTED;
    if (!X || !qweight || !scales || !Y) return W4_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(qweight, 16) || !aligned(scales, 16) || !aligned(zeros, 16) ||
        !aligned(g_idx, 16) || !aligned(s_inv, 16) || !aligned(Y, 16) || !aligned(workspace, 256))
        return W4_ERR_INVALID_ARG;
    const bool bf16 = act_dtype == W4_BF16;
    const bool gidx = g_idx != nullptr;
    if (bf16 && gidx) return W4_ERR_UNSUPPORTED;
    const size_t need = w4a16_workspace_bytes(M, N, K, group_size);
    if (need == 0) return W4_ERR_CUDA;
    const bool prefill = M > kDecodeMaxM;
    if (perm && (prefill || !decode_x_resident(M, K))) return W4_ERR_UNSUPPORTED;
    const bool needs_ws = !prefill || s_inv != nullptr;
    if (needs_ws && (!workspace || workspace_bytes < need)) return W4_ERR_INVALID_ARG;
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return W4_ERR_CUDA;
    cudaStream_t strm = as_stream(stream);

    if (!prefill) {
        w4d::DecodeParams p;
        std::memset(&p, 0, sizeof(p));
        p.qw = qweight;
        p.scales = reinterpret_cast<const __half*>(scales);
        p.zeros = reinterpret_cast<const __half*>(zeros);
        p.g_idx = g_idx;
        p.s_inv = s_inv;
        p.perm = perm;
        p.Y = Y;
        p.M = (int)M;
        p.N = (int)N;
        p.K = (int)K;
        p.group_size = group_size;
        p.G = (int)(K / group_size);
        p.out_dtype = (int)out_dtype;
        p.KA = (int)(K / 64);
        p.tiles = (int)(N / 16);
        unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
        const int mode = decode_mode(K, group_size, gidx);
        const size_t pre_off = pre_offset(8, sm_count(dev));
        if (bf16) return dispatch_decode<true>(mode, p, X, ws, pre_off, dev, strm);
        return dispatch_decode<false>(mode, p, X, ws, pre_off, dev, strm);
    }

    const void* Xeff = X;
    if (s_inv) {
        const size_t pairs = (size_t)M * (size_t)K / 2;
        const unsigned blocks = (unsigned)((pairs + 255) / 256 < 65535 * 8 ? (pairs + 255) / 256 : 65535 * 8);
        void* xp = reinterpret_cast<unsigned char*>(workspace) + kCounterBytes + slot_region_bytes(sm_count(dev));
        if (bf16) w4p::scale_acts_kernel<true><<<blocks, 256, 0, strm>>>(X, s_inv, xp, (int)M, (int)K);
        else w4p::scale_acts_kernel<false><<<blocks, 256, 0, strm>>>(X, s_inv, xp, (int)M, (int)K);
        if (cudaGetLastError() != cudaSuccess) return W4_ERR_CUDA;
        Xeff = xp;
    }
    CUtensorMap map;
    if (!make_act_tensor_map(&map, Xeff, bf16, M, K, w4p::BM)) return W4_ERR_CUDA;
    w4p::PrefillParams p;
    std::memset(&p, 0, sizeof(p));
    p.qw = qweight;
    p.scales = reinterpret_cast<const __half*>(scales);
    p.zeros = reinterpret_cast<const __half*>(zeros);
    p.g_idx = g_idx;
    p.Y = Y;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.group_size = group_size;
    p.G = (int)(K / group_size);
    p.out_dtype = (int)out_dtype;
    p.KA = (int)(K / 64);
    p.tiles = (int)(N / 16);
    if (bf16) return launch_prefill<true, w4p::kWInt4>(map, p, dev, strm);
    return gidx ? launch_prefill<false, w4p::kWGidx>(map, p, dev, strm)
                : launch_prefill<false, w4p::kWInt4>(map, p, dev, strm);
}

size_t w4a16_workspace_bytes_perm(int64_t M, int64_t N, int64_t K, int32_t group_size) {
    if (M < 0 || check_layer_shape(N, K, group_size) != W4_OK) return 0;
    if (M == 0) return 0;
    const int dev = current_device();
    const int sms = dev >= 0 ? sm_count(dev) : 0;
    if (sms <= 0) return 0;
    // the gathered activations sit behind everything the GEMM itself uses
    return perm_gather_offset(M, K, sms) + (size_t)(((size_t)M * (size_t)K * 2 + 255) / 256 * 256);
}

w4_status w4a16_gemm_perm(const void* X, w4_dtype act_dtype, int64_t M, int64_t N, int64_t K,
                          const uint32_t* qweight, const void* scales, const void* zeros,
                          const int32_t* perm, int32_t group_size, const float* s_inv, void* Y,
                          w4_dtype out_dtype, void* workspace, size_t workspace_bytes,
                          w4_stream_t stream) {
    if (M < 0) return W4_ERR_INVALID_ARG;
    if (act_dtype != W4_F16 && act_dtype != W4_BF16) return W4_ERR_INVALID_ARG;
    w4_status st = check_layer_shape(N, K, group_size);
    if (st != W4_OK) return st;
    if (M == 0) return W4_OK;
    if (M > INT_MAX / 2 || (size_t)M * (size_t)K > (size_t)INT_MAX * 8) return W4_ERR_UNSUPPORTED;
    if (!X || !perm || !workspace) return W4_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(perm, 16) || !aligned(s_inv, 16) || !aligned(workspace, 256))
        return W4_ERR_INVALID_ARG;
    const size_t need = w4a16_workspace_bytes_perm(M, N, K, group_size);
    if (need == 0) return W4_ERR_CUDA;
    if (workspace_bytes < need) return W4_ERR_INVALID_ARG;
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return W4_ERR_CUDA;
    if (M <= kDecodeMaxM && decode_x_resident(M, K))   // the decode kernel gathers while preparing X'
        return gemm_impl(X, act_dtype, M, N, K, qweight, scales, zeros, nullptr, perm, group_size, s_inv, Y,
                         out_dtype, workspace, workspace_bytes, stream);
    cudaStream_t strm = as_stream(stream);
    void* xp = reinterpret_cast<unsigned char*>(workspace) + perm_gather_offset(M, K, sm_count(dev));
    const size_t chunks = (size_t)M * (size_t)K / 8;
    const unsigned blocks = (unsigned)std::min<size_t>((chunks + 255) / 256, (size_t)65535 * 8);
    if (act_dtype == W4_BF16) w4a::gather_acts_kernel<true><<<blocks, 256, 0, strm>>>(X, perm, s_inv, xp, (int)M, (int)K);
    else w4a::gather_acts_kernel<false><<<blocks, 256, 0, strm>>>(X, perm, s_inv, xp, (int)M, (int)K);
    if (cudaGetLastError() != cudaSuccess) return W4_ERR_CUDA;
    // the contiguous-group GEMM on the gathered, already scaled activations
    return gemm_impl(xp, act_dtype, M, N, K, qweight, scales, zeros, nullptr, nullptr, group_size, nullptr, Y,
                     out_dtype, workspace, workspace_bytes, stream);
}

size_t w4_awq_search_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t group_size,
                                     int32_t symmetric, int32_t n_grid) {
    if (M <= 0 || M > kAwqMaxRows || n_grid <= 0 || n_grid > 1024) return 0;
    if (check_layer_shape(N, K, group_size) != W4_OK) return 0;
    const size_t gemm = w4a16_workspace_bytes(M, N, K, group_size);
    if (gemm == 0) return 0;
    return awq_layout(M, N, K, group_size, symmetric, n_grid, gemm).total;
}

w4_status w4_awq_search(const void* W, w4_dtype w_dtype, int64_t N, int64_t K, const void* X,
                        w4_dtype x_dtype, int64_t M, int32_t group_size, int32_t symmetric,
                        int32_t n_grid, float* s_best, double* losses, int32_t* best,
                        void* workspace, size_t workspace_bytes, w4_stream_t stream) {
    if (!W || !X || !s_best || !losses || !best || !workspace) return W4_ERR_INVALID_ARG;
    if ((w_dtype != W4_F16 && w_dtype != W4_BF16) || (x_dtype != W4_F16 && x_dtype != W4_BF16))
        return W4_ERR_INVALID_ARG;
    if (symmetric != 0 && symmetric != 1) return W4_ERR_INVALID_ARG;
    if (M <= 0 || M > kAwqMaxRows || n_grid <= 0 || n_grid > 1024) return W4_ERR_INVALID_ARG;
    w4_status st = check_layer_shape(N, K, group_size);
    if (st != W4_OK) return st;
    if (K / group_size > kQuantMaxGroups) return W4_ERR_UNSUPPORTED;
    if (!aligned(W, 16) || !aligned(X, 16) || !aligned(s_best, 4) || !aligned(workspace, 256))
        return W4_ERR_INVALID_ARG;
    const size_t gemm_bytes = w4a16_workspace_bytes(M, N, K, group_size);
    if (gemm_bytes == 0) return W4_ERR_CUDA;
    const AwqLayout L = awq_layout(M, N, K, group_size, symmetric, n_grid, gemm_bytes);
    if (workspace_bytes < L.total) return W4_ERR_INVALID_ARG;
    cudaStream_t strm = as_stream(stream);
    unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
    double* logm = reinterpret_cast<double*>(ws + L.logm);
    double* mu = reinterpret_cast<double*>(ws + L.mu);
    float* s = reinterpret_cast<float*>(ws + L.s);
    float* s_inv = reinterpret_cast<float*>(ws + L.s_inv);
    uint32_t* qw = reinterpret_cast<uint32_t*>(ws + L.qw);
    void* sc = ws + L.sc;
    void* zr = symmetric ? nullptr : (void*)(ws + L.zr);
    float* yref = reinterpret_cast<float*>(ws + L.yref);
    float* yq = reinterpret_cast<float*>(ws + L.yq);
    double* part = reinterpret_cast<double*>(ws + L.part);
    double* loss = reinterpret_cast<double*>(ws + L.loss);
    const bool xb = x_dtype == W4_BF16, wb = w_dtype == W4_BF16;
    const unsigned kb = (unsigned)((K + 255) / 256);
    // activation statistics and the unquantised reference product, once
    if (xb) w4s::col_logmean_kernel<true><<<kb, 256, 0, strm>>>(X, (int)M, (int)K, logm);
    else w4s::col_logmean_kernel<false><<<kb, 256, 0, strm>>>(X, (int)M, (int)K, logm);
    w4s::mean_kernel<<<1, 32, 0, strm>>>(logm, (int)K, mu);
    const dim3 rb(w4s::kT, w4s::kT), rg((unsigned)((N + w4s::kT - 1) / w4s::kT), (unsigned)((M + w4s::kT - 1) / w4s::kT));
    if (xb && wb) w4s::ref_gemm_kernel<true, true><<<rg, rb, 0, strm>>>(X, W, (int)M, (int)N, (int)K, yref);
    else if (xb) w4s::ref_gemm_kernel<true, false><<<rg, rb, 0, strm>>>(X, W, (int)M, (int)N, (int)K, yref);
    else if (wb) w4s::ref_gemm_kernel<false, true><<<rg, rb, 0, strm>>>(X, W, (int)M, (int)N, (int)K, yref);
    else w4s::ref_gemm_kernel<false, false><<<rg, rb, 0, strm>>>(X, W, (int)M, (int)N, (int)K, yref);
    if (cudaGetLastError() != cudaSuccess) return W4_ERR_CUDA;
    const size_t n = (size_t)M * (size_t)N;
    const size_t chunk = (n + L.nblk - 1) / L.nblk;
    for (int j = 0; j < n_grid; ++j) {
        const double a = (double)j / (double)n_grid;
        w4s::awq_scale_kernel<<<kb, 256, 0, strm>>>(logm, mu, a, (int)K, s, s_inv);
        if (cudaGetLastError() != cudaSuccess) return W4_ERR_CUDA;
        st = quantize_pack_impl(W, w_dtype, N, K, s, group_size, symmetric, nullptr, nullptr, qw, sc, zr, stream);
        if (st != W4_OK) return st;
        st = gemm_impl(X, x_dtype, M, N, K, qw, sc, zr, nullptr, nullptr, group_size, s_inv, yq, W4_F32,
                       ws + L.gemm, workspace_bytes - L.gemm, stream);
        if (st != W4_OK) return st;
        w4s::sqdiff_partial_kernel<<<(unsigned)L.nblk, w4s::kLossThreads, 0, strm>>>(yref, yq, n, chunk, part);
        w4s::sum_kernel<<<1, 32, 0, strm>>>(part, L.nblk, loss + j);
        if (cudaGetLastError() != cudaSuccess) return W4_ERR_CUDA;
    }
    if (cudaMemcpyAsync(losses, loss, (size_t)n_grid * sizeof(double), cudaMemcpyDeviceToHost, strm) != cudaSuccess ||
        cudaStreamSynchronize(strm) != cudaSuccess)
        return W4_ERR_CUDA;
    int b = 0;
    for (int j = 1; j < n_grid; ++j)
        if (losses[j] < losses[b]) b = j;   // the first of equal losses
    *best = b;
    w4s::awq_scale_kernel<<<kb, 256, 0, strm>>>(logm, mu, (double)b / (double)n_grid, (int)K, s_best, s_inv);
    if (cudaGetLastError() != cudaSuccess || cudaStreamSynchronize(strm) != cudaSuccess) return W4_ERR_CUDA;
    return W4_OK;
}

w4_status w4_unpack_canonical(const uint32_t* qweight, int64_t N, int64_t K,
                              uint32_t* qweight_canonical, w4_stream_t stream) {
    if (!qweight || !qweight_canonical) return W4_ERR_INVALID_ARG;
    if (!aligned(qweight, 4) || !aligned(qweight_canonical, 4)) return W4_ERR_INVALID_ARG;
    w4_status st = check_layer_shape(N, K, 64);
    if (st != W4_OK) return st;
    const size_t total = (size_t)N * (size_t)(K / 8);
    const unsigned blocks = (unsigned)((total + 255) / 256 < 65535 * 16 ? (total + 255) / 256 : 65535 * 16);
    w4q::unpack_canonical_kernel<<<blocks, 256, 0, as_stream(stream)>>>(qweight, (int)N, (int)K,
                                                                       qweight_canonical);
    return launch_status();
}

w4_status w4_check_device_error(void) {
    if (cudaDeviceSynchronize() != cudaSuccess) return W4_ERR_CUDA;
    unsigned word = 0;
    if (cudaMemcpyFromSymbol(&word, g_w4_error_word, sizeof(word)) != cudaSuccess) return W4_ERR_CUDA;
    if (word != 0) {
        const unsigned zero = 0;
        if (cudaMemcpyToSymbol(g_w4_error_word, &zero, sizeof(zero)) != cudaSuccess) return W4_ERR_CUDA;
    }
    // A kernel that gave up a wait may have left split-K flags set in the scratch it used.
    // The library's own allocation-free scratch is zeroed again here (every kernel has
    // finished after the synchronisation above); a caller's workspace is the caller's to
    // zero.
    if ((word & W4_DEVERR_TIMEOUT) && noalloc_rezero(current_device()) != cudaSuccess) return W4_ERR_CUDA;
    if (word & W4_DEVERR_TIMEOUT) return W4_ERR_TIMEOUT;
    if (word & W4_DEVERR_GIDX) return W4_ERR_DEVICE_ARG;
    return W4_OK;
}

w4_status w4_set_wait_limit_ns(uint64_t ns) {
    unsigned long long v = ns < 1000 ? 1000ull : (unsigned long long)ns;
    return cudaMemcpyToSymbol(g_w4_wait_limit_ns, &v, sizeof(v)) == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

}  // extern "C"

namespace {
// One thread waits on a barrier nothing will complete; the bounded wait expires.
__global__ void expired_wait_kernel() {
    __shared__ uint64_t bar;
    if (threadIdx.x == 0) {
        mbar_init(&bar, 1);
        fence_mbar_init();
        (void)mbar_wait(&bar, 0);
    }
}
}  // namespace

extern "C" w4_status w4_selftest_expired_wait(w4_stream_t stream) {
    expired_wait_kernel<<<1, 32, 0, as_stream(stream)>>>();
    return launch_status();
}

// ---------------------------------------------------------------------------------------
// w4a16_gemm_noalloc: the small-batch GEMM for callers that cannot hand the library a
// workspace.  Its scratch (split-K counters and partial sums) is one fixed array in
// device memory that exists on every GPU that loads this library, from module load to
// process exit.  Host code never dereferences the array's name: it is only a host-side
// handle, so the device address is fetched once per device with cudaGetSymbolAddress.
// ---------------------------------------------------------------------------------------
namespace {

constexpr size_t kNoAllocScratchBytes = (size_t)8 << 20;   // 8 MiB
constexpr int kNoAllocMaxTiles = 4;                          // token tiles: M <= 32
__device__ __align__(256) unsigned char g_w4_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocScratch {
    std::mutex mu;
    void* ptr = nullptr;   // set once the set-up has succeeded; a failed set-up is retried
};
NoAllocScratch g_noalloc[kMaxDevices];

// Set-up on the first successful call per device (that device current): look up the
// array's device address and zero it (every call expects the split-K flags it reads to
// start at zero and leaves them at zero).  A failed set-up leaves ptr null, so the next
// call tries again.
void* noalloc_scratch(int dev) {
    NoAllocScratch& s = g_noalloc[dev];
    std::lock_guard<std::mutex> lock(s.mu);
    if (s.ptr) return s.ptr;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_w4_noalloc_scratch) != cudaSuccess) return nullptr;
    if (cudaMemset(p, 0, kNoAllocScratchBytes) != cudaSuccess) return nullptr;
    if (cudaDeviceSynchronize() != cudaSuccess) return nullptr;
    s.ptr = p;
    return p;
}

cudaError_t noalloc_rezero(int dev) {
    if (dev < 0 || dev >= kMaxDevices) return cudaSuccess;
    NoAllocScratch& s = g_noalloc[dev];
    std::lock_guard<std::mutex> lock(s.mu);
    if (!s.ptr) return cudaSuccess;   // never set up: nothing was used
    cudaError_t e = cudaMemset(s.ptr, 0, kNoAllocScratchBytes);
    if (e == cudaSuccess) e = cudaDeviceSynchronize();
    return e;
}

// Test aid: every split-K word of the scratch set to a flagged partial of 1.0, or the
// nonzero words counted.
__device__ unsigned long long g_w4_selftest_count;

__global__ void plant_stale_kernel(unsigned long long* words, size_t n) {
    const unsigned long long w = (1ull << 32) | (unsigned long long)__float_as_uint(1.0f);
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        words[i] = w;
}

__global__ void count_nonzero_kernel(const unsigned long long* words, size_t n) {
    unsigned long long c = 0;
    for (size_t i = blockIdx.x * (size_t)blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
        c += words[i] != 0ull;
    if (c) atomicAdd(&g_w4_selftest_count, c);
}

}  // namespace

extern "C" w4_status w4_selftest_noalloc_scratch(int32_t plant, uint64_t* nonzero_words) {
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return W4_ERR_CUDA;
    if (!plant && !nonzero_words) return W4_ERR_INVALID_ARG;
    unsigned char* ws = reinterpret_cast<unsigned char*>(noalloc_scratch(dev));
    if (!ws) return W4_ERR_CUDA;
    unsigned long long* words = reinterpret_cast<unsigned long long*>(ws + kCounterBytes);
    const int sms = sm_count(dev);
    if (sms <= 0) return W4_ERR_CUDA;
    const size_t n = decode_slot_bytes(kNoAllocMaxTiles, sms) / 8;   // the split-K slot region
    if (plant) {
        plant_stale_kernel<<<256, 256>>>(words, n);
        if (cudaGetLastError() != cudaSuccess || cudaDeviceSynchronize() != cudaSuccess) return W4_ERR_CUDA;
        if (nonzero_words) *nonzero_words = n;
        return W4_OK;
    }
    const unsigned long long zero = 0;
    if (cudaMemcpyToSymbol(g_w4_selftest_count, &zero, sizeof(zero)) != cudaSuccess) return W4_ERR_CUDA;
    count_nonzero_kernel<<<256, 256>>>(words, n);
    unsigned long long c = 0;
    if (cudaGetLastError() != cudaSuccess || cudaMemcpyFromSymbol(&c, g_w4_selftest_count, sizeof(c)) != cudaSuccess)
        return W4_ERR_CUDA;
    *nonzero_words = c;
    return W4_OK;
}

extern "C" w4_status w4a16_gemm_noalloc(const void* X, w4_dtype act_dtype, int64_t M, int64_t N,
                                        int64_t K, const uint32_t* qweight, const void* scales,
                                        const void* zeros, const int32_t* g_idx, int32_t group_size,
                                        const float* s_inv, void* Y, w4_dtype out_dtype,
                                        w4_stream_t stream) {
    if (M < 0) return W4_ERR_INVALID_ARG;
    if (act_dtype != W4_F16 && act_dtype != W4_BF16) return W4_ERR_INVALID_ARG;
    if (out_dtype != W4_F16 && out_dtype != W4_BF16 && out_dtype != W4_F32) return W4_ERR_INVALID_ARG;
    w4_status st = check_layer_shape(N, K, group_size);
    if (st != W4_OK) return st;
    if (M == 0) return W4_OK;
    if (M > kDecodeMaxM) return W4_ERR_UNSUPPORTED;
    if (!X || !qweight || !scales || !Y) return W4_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(qweight, 16) || !aligned(scales, 16) || !aligned(zeros, 16) ||
        !aligned(g_idx, 16) || !aligned(s_inv, 16) || !aligned(Y, 16))
        return W4_ERR_INVALID_ARG;
    const bool bf16 = act_dtype == W4_BF16;
    const bool gidx = g_idx != nullptr;
    if (bf16 && gidx) return W4_ERR_UNSUPPORTED;
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return W4_ERR_CUDA;
    const int sms = sm_count(dev);
    if (sms <= 0) return W4_ERR_CUDA;
    if (decode_tiles_for(M) > kNoAllocMaxTiles ||
        decode_workspace_bytes(M, K, sms, kNoAllocMaxTiles) > kNoAllocScratchBytes)
        return W4_ERR_UNSUPPORTED;
    unsigned char* ws = reinterpret_cast<unsigned char*>(noalloc_scratch(dev));
    if (!ws) return W4_ERR_CUDA;

    w4d::DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.qw = qweight;
    p.scales = reinterpret_cast<const __half*>(scales);
    p.zeros = reinterpret_cast<const __half*>(zeros);
    p.g_idx = g_idx;
    p.s_inv = s_inv;
    p.Y = Y;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.group_size = group_size;
    p.G = (int)(K / group_size);
    p.out_dtype = (int)out_dtype;
    p.KA = (int)(K / 64);
    p.tiles = (int)(N / 16);
    cudaStream_t strm = as_stream(stream);
    const int mode = decode_mode(K, group_size, gidx);
    const size_t pre_off = pre_offset(kNoAllocMaxTiles, sms);
    if (bf16) return dispatch_decode<true>(mode, p, X, ws, pre_off, dev, strm);
    return dispatch_decode<false>(mode, p, X, ws, pre_off, dev, strm);
}

// ---------------------------------------------------------------------------------------
// w4a16_gemm_chain: a list of decode GEMMs (M <= 8, one token tile, X' resident) in
// persistent launches of up to w4c::kMaxLayers layers each.
// ---------------------------------------------------------------------------------------
namespace {

size_t chain_workspace_bytes(int sms) { return kCounterBytes + decode_slot_bytes(1, sms); }

// The layer-sequence kernel keeps every layer's X' and sums resident; up to 120 KB of them
// still leave the weight ring at least three stages (checked again per launch).
bool chain_x_resident(int64_t M, int64_t K) {
    auto up = [](int64_t v, int64_t a) { return (v + a - 1) / a * a; };
    if (M > 8) return false;
    const int64_t sstride = std::max<int64_t>(2, (M + 1) / 2 * 2);
    return up(M * K * 2, 128) + up((K / 32 + K / 64 + K / 128) * sstride * 4, 128) <= 120 * 1024;
}

template <bool BF16, int MODE>
w4_status launch_chain(w4c::ChainParams& cp, int smem, int grid, int dev, cudaStream_t stream) {
    static std::once_flag flags[kMaxDevices];
    auto k = w4c::chain_kernel<BF16, MODE>;
    bool attr_ok = true;
    std::call_once(flags[dev], [&] {
        attr_ok = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) ==
                  cudaSuccess;
    });
    if (!attr_ok) return W4_ERR_CUDA;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)grid);
    cfg.blockDim = dim3(w4d::Cfg<1>::threads);
    cfg.dynamicSmemBytes = (size_t)smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaLaunchKernelEx(&cfg, k, cp) != cudaSuccess) return W4_ERR_CUDA;
    return launch_status();
}

// One launch over layers [l0, l0 + n) of the list (n <= kMaxLayers).
w4_status chain_launch(const w4_chain_layer* layers, int l0, int n, int M, bool bf16, int out_dtype, int mode,
                       unsigned char* ws, int dev, int sms, cudaStream_t stream) {
    using C = w4d::Cfg<1>;
    auto up = [](int v, int a) { return (v + a - 1) / a * a; };
    constexpr int kMaxSmem = 227 * 1024;
    // ring geometry shared by the launch's layers: codes | scale rows | zero-point rows |
    // stage descriptor, sized for the largest per-stage group-row count
    const int span = 64 * C::aps;
    int ngs_max = 1, kmax = 64;
    bool any_zeros = false;
    for (int l = l0; l < l0 + n; ++l) {
        const int g = layers[l].group_size;
        const int G = (int)(layers[l].K / g);
        const int ngs = g == 32 ? span / 32 : std::min(G, (span + 2 * g - 65) / g);
        ngs_max = std::max(ngs_max, ngs);
        kmax = std::max(kmax, (int)layers[l].K);
        any_zeros = any_zeros || layers[l].zeros != nullptr;
    }
    const int sstride = std::max(2, (M + 1) / 2 * 2);
    const int res_x = up(M * kmax * 2, 128);
    const int res_s = up((kmax / 32 + kmax / 64 + kmax / 128) * sstride * 4, 128);
    const int off_sc = C::aps * w4d::kTilesPerBand * 512;
    const int off_zr = off_sc + ngs_max * 256;
    const int off_desc = off_zr + (any_zeros ? ngs_max * 256 : 0);
    const int stage_bytes = up(off_desc + 48, 1024);
    const int fixed = res_x + res_s + C::xchg_bytes + 3 * w4d::kMaxStages * 8 + 16 + 1024;
    const int stages = std::min(w4d::kMaxStages, (kMaxSmem - fixed) / stage_bytes);
    if (stages < 3) return W4_ERR_UNSUPPORTED;
    const int smem = stages * stage_bytes + fixed;

    static w4c::ChainParams cp_storage[kMaxDevices];   // large: kept off the stack
    static std::mutex cp_mu[kMaxDevices];
    std::lock_guard<std::mutex> lock(cp_mu[dev]);
    w4c::ChainParams& cp = cp_storage[dev];
    std::memset(&cp, 0, sizeof(cp));
    cp.n_layers = n;
    cp.counter = reinterpret_cast<unsigned int*>(ws);   // word 0 of the zero region
    for (int j = 0; j < n; ++j) {
        const w4_chain_layer& Lc = layers[l0 + j];
        w4d::DecodeParams& p = cp.L[j];
        p.qw = Lc.qweight;
        p.scales = reinterpret_cast<const __half*>(Lc.scales);
        p.zeros = reinterpret_cast<const __half*>(Lc.zeros);
        p.s_inv = Lc.s_inv;
        p.X = Lc.X;
        p.Y = Lc.Y;
        p.slots = reinterpret_cast<unsigned long long*>(ws + kCounterBytes);
        p.M = M;
        p.N = (int)Lc.N;
        p.K = (int)Lc.K;
        p.ldx = (int)Lc.ldx;
        p.group_size = Lc.group_size;
        p.G = (int)(Lc.K / Lc.group_size);
        p.out_dtype = out_dtype;
        p.KA = (int)(Lc.K / 64);
        p.KU = (p.KA + 1) / 2;
        p.tiles = (int)(Lc.N / 16);
        const int bands = (p.tiles + w4d::kTilesPerBand - 1) / w4d::kTilesPerBand;
        p.units = bands * p.KU;
        p.base = p.units / sms;
        p.rem = p.units % sms;
        const int g = p.group_size;
        p.ngs = g == 32 ? span / 32 : std::min(p.G, (span + 2 * g - 65) / g);
        p.srow_bytes = 256;
        p.stages = stages;
        p.xres = 1;
        p.sstride = sstride;
        p.off_x = p.off_xs = p.off_sx = p.off_si = off_sc;
        p.off_sc = off_sc;
        p.off_zr = off_zr;
        p.off_gi = off_desc;
        p.off_desc = off_desc;
        p.stage_bytes = stage_bytes;
        p.off_res = stages * stage_bytes;
        p.off_res_s = p.off_res + res_x;
        p.off_xchg = p.off_res + res_x + res_s;
        if (!make_meta_map(&cp.sc[j], p.scales, p.G, p.N, p.ngs)) return W4_ERR_CUDA;
        if (p.zeros && !make_meta_map(&cp.zr[j], p.zeros, p.G, p.N, p.ngs)) return W4_ERR_CUDA;
        if (!p.zeros) cp.zr[j] = cp.sc[j];
    }
    if (bf16) {
        if (mode == w4d::kModeHalf) return launch_chain<true, w4d::kModeHalf>(cp, smem, sms, dev, stream);
        if (mode == w4d::kModeG32) return launch_chain<true, w4d::kModeG32>(cp, smem, sms, dev, stream);
        return launch_chain<true, w4d::kModeAtom>(cp, smem, sms, dev, stream);
    }
    if (mode == w4d::kModeHalf) return launch_chain<false, w4d::kModeHalf>(cp, smem, sms, dev, stream);
    if (mode == w4d::kModeG32) return launch_chain<false, w4d::kModeG32>(cp, smem, sms, dev, stream);
    return launch_chain<false, w4d::kModeAtom>(cp, smem, sms, dev, stream);
}

}  // namespace

extern "C" size_t w4a16_chain_workspace_bytes(int64_t M) {
    if (M < 1 || M > 8) return 0;
    const int dev = current_device();
    const int sms = dev >= 0 ? sm_count(dev) : 0;
    return sms > 0 ? chain_workspace_bytes(sms) : 0;
}

extern "C" w4_status w4a16_gemm_chain(const w4_chain_layer* layers, int32_t n_layers, int64_t M,
                                      w4_dtype act_dtype, w4_dtype out_dtype, void* workspace,
                                      size_t workspace_bytes, w4_stream_t stream) {
    if (!layers || n_layers < 0 || M < 0) return W4_ERR_INVALID_ARG;
    if (act_dtype != W4_F16 && act_dtype != W4_BF16) return W4_ERR_INVALID_ARG;
    if (out_dtype != W4_F16 && out_dtype != W4_BF16 && out_dtype != W4_F32) return W4_ERR_INVALID_ARG;
    if (n_layers == 0 || M == 0) return W4_OK;
    if (M > 8) return W4_ERR_UNSUPPORTED;
    int mode = -1;
    for (int l = 0; l < n_layers; ++l) {
        const w4_chain_layer& L = layers[l];
        w4_status st = check_layer_shape(L.N, L.K, L.group_size);
        if (st != W4_OK) return st;
        if (!L.X || !L.qweight || !L.scales || !L.Y) return W4_ERR_INVALID_ARG;
        if (!aligned(L.X, 16) || !aligned(L.qweight, 16) || !aligned(L.scales, 16) || !aligned(L.zeros, 16) ||
            !aligned(L.s_inv, 16) || !aligned(L.Y, 16))
            return W4_ERR_INVALID_ARG;
        if (L.ldx < L.K || L.ldx % 8 != 0 || L.ldx > INT_MAX / 16) return W4_ERR_INVALID_ARG;
        if (!chain_x_resident(M, L.K)) return W4_ERR_UNSUPPORTED;
        const int m = decode_mode(L.K, L.group_size, false);
        if (mode >= 0 && m != mode) return W4_ERR_UNSUPPORTED;   // one group mode per list
        mode = m;
    }
    if (!aligned(workspace, 256)) return W4_ERR_INVALID_ARG;
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return W4_ERR_CUDA;
    const int sms = sm_count(dev);
    if (sms <= 0) return W4_ERR_CUDA;
    if (!workspace || workspace_bytes < chain_workspace_bytes(sms)) return W4_ERR_INVALID_ARG;
    unsigned char* ws = reinterpret_cast<unsigned char*>(workspace);
    cudaStream_t strm = as_stream(stream);
    for (int l0 = 0; l0 < n_layers; l0 += w4c::kMaxLayers) {
        const int n = std::min(w4c::kMaxLayers, n_layers - l0);
        w4_status st = chain_launch(layers, l0, n, (int)M, act_dtype == W4_BF16, (int)out_dtype, mode, ws, dev,
                                    sms, strm);
        if (st != W4_OK) return st;
    }
    return W4_OK;
}

// ---------------------------------------------------------------------------------------
// Block-scaled FP4 weights (NVFP4, MXFP4): quantise/pack, and the GEMM with 16-bit
// activations (the decode kernel's FP4 modes for M <= 64, the prefill kernel above).
// ---------------------------------------------------------------------------------------
namespace {

int fp4_block(w4_fp4_format f) { return f == W4_FP4_NVFP4 ? 16 : 32; }

w4_status check_fp4_shape(int64_t N, int64_t K) {
    if (N <= 0 || K <= 0) return W4_ERR_INVALID_ARG;
    if (N > INT_MAX / 2 || K > INT_MAX / 2) return W4_ERR_UNSUPPORTED;
    if (N % 16 != 0 || K % 64 != 0 || N > kMaxBands * 128) return W4_ERR_UNSUPPORTED;
    return W4_OK;
}

template <int FMT, bool BF16W>
w4_status launch_fp4_pack(const w4f::Fp4Params& p, int dev, cudaStream_t s) {
    static std::once_flag flags[kMaxDevices];
    const int smem = (p.K / w4f::Fmt<FMT>::block) * w4f::kRows;
    if (!ensure_smem(w4f::fp4_pack_kernel<FMT, BF16W>, 227 * 1024, flags, dev)) return W4_ERR_CUDA;
    w4f::fp4_pack_kernel<FMT, BF16W><<<(unsigned)(p.N / 16), w4f::kThreads, smem, s>>>(p);
    return launch_status();
}

}  // namespace

extern "C" w4_status w4_fp4_quantize_pack(const void* W, w4_dtype w_dtype, int64_t N, int64_t K,
                                          w4_fp4_format format, uint32_t* qweight, uint8_t* block_scales,
                                          float* tensor_scale, w4_stream_t stream) {
    if (!W || !qweight || !block_scales) return W4_ERR_INVALID_ARG;
    if (w_dtype != W4_F16 && w_dtype != W4_BF16) return W4_ERR_INVALID_ARG;
    if (format != W4_FP4_NVFP4 && format != W4_FP4_MXFP4) return W4_ERR_INVALID_ARG;
    if ((format == W4_FP4_NVFP4) != (tensor_scale != nullptr)) return W4_ERR_INVALID_ARG;
    if (!aligned(W, 2) || !aligned(qweight, 4) || !aligned(tensor_scale, 4)) return W4_ERR_INVALID_ARG;
    w4_status st = check_fp4_shape(N, K);
    if (st != W4_OK) return st;
    if ((K / fp4_block(format)) * w4f::kRows > 227 * 1024) return W4_ERR_UNSUPPORTED;
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return W4_ERR_CUDA;
    cudaStream_t strm = as_stream(stream);
    w4f::Fp4Params p;
    p.W = W;
    p.qweight = qweight;
    p.bscale = block_scales;
    p.tscale = tensor_scale;
    p.N = (int)N;
    p.K = (int)K;
    const bool bf16 = w_dtype == W4_BF16;
    if (format == W4_FP4_NVFP4) {
        // the tensor's amax (into *tensor_scale), the packing, then gs in its place
        if (cudaMemsetAsync(tensor_scale, 0, sizeof(float), strm) != cudaSuccess) return W4_ERR_CUDA;
        const size_t n = (size_t)N * (size_t)K;
        const unsigned blocks = (unsigned)std::min<size_t>((n + 255) / 256, (size_t)sm_count(dev) * 8);
        if (bf16) w4f::amax_kernel<true><<<blocks, 256, 0, strm>>>(W, n, tensor_scale);
        else w4f::amax_kernel<false><<<blocks, 256, 0, strm>>>(W, n, tensor_scale);
        if (cudaGetLastError() != cudaSuccess) return W4_ERR_CUDA;
        st = bf16 ? launch_fp4_pack<w4f::kNvfp4, true>(p, dev, strm) : launch_fp4_pack<w4f::kNvfp4, false>(p, dev, strm);
        if (st != W4_OK) return st;
        w4f::finish_tscale_kernel<<<1, 1, 0, strm>>>(tensor_scale);
        return launch_status();
    }
    return bf16 ? launch_fp4_pack<w4f::kMxfp4, true>(p, dev, strm) : launch_fp4_pack<w4f::kMxfp4, false>(p, dev, strm);
}

extern "C" size_t w4a16_fp4_workspace_bytes(int64_t M, int64_t N, int64_t K, w4_fp4_format format) {
    if (format != W4_FP4_NVFP4 && format != W4_FP4_MXFP4) return 0;
    if (M <= 0 || check_fp4_shape(N, K) != W4_OK) return 0;
    const int dev = current_device();
    const int sms = dev >= 0 ? sm_count(dev) : 0;
    if (sms <= 0) return 0;
    if (M <= kDecodeMaxM) return decode_workspace_bytes(M, K, sms);
    return 0;   // the prefill kernel needs no workspace
}

extern "C" w4_status w4a16_fp4_gemm(const void* X, w4_dtype act_dtype, int64_t M, int64_t N, int64_t K,
                                    const uint32_t* qweight, const uint8_t* block_scales,
                                    const float* tensor_scale, w4_fp4_format format, void* Y,
                                    w4_dtype out_dtype, void* workspace, size_t workspace_bytes,
                                    w4_stream_t stream) {
    if (M < 0) return W4_ERR_INVALID_ARG;
    if (format != W4_FP4_NVFP4 && format != W4_FP4_MXFP4) return W4_ERR_INVALID_ARG;
    if (act_dtype != W4_F16 && act_dtype != W4_BF16) return W4_ERR_INVALID_ARG;
    if (out_dtype != W4_F16 && out_dtype != W4_BF16 && out_dtype != W4_F32) return W4_ERR_INVALID_ARG;
    w4_status st = check_fp4_shape(N, K);
    if (st != W4_OK) return st;
    if (M == 0) return W4_OK;
    if (act_dtype != W4_F16) return W4_ERR_UNSUPPORTED;   // E2M1 decodes exactly to fp16
    if (!X || !qweight || !block_scales || !Y) return W4_ERR_INVALID_ARG;
    if ((format == W4_FP4_NVFP4) != (tensor_scale != nullptr)) return W4_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(qweight, 16) || !aligned(block_scales, 16) || !aligned(Y, 16) ||
        !aligned(tensor_scale, 4) || !aligned(workspace, 256))
        return W4_ERR_INVALID_ARG;
    if (M > INT_MAX / 2 || (size_t)M * (size_t)K > (size_t)INT_MAX * 8) return W4_ERR_UNSUPPORTED;
    const int dev = current_device();
    if (dev < 0 || dev >= kMaxDevices) return W4_ERR_CUDA;
    const int B = fp4_block(format);
    cudaStream_t strm = as_stream(stream);
    if (M > kDecodeMaxM) {
        CUtensorMap map;
        if (!make_act_tensor_map(&map, X, false, M, K, w4p::BM)) return W4_ERR_CUDA;
        w4p::PrefillParams pp;
        std::memset(&pp, 0, sizeof(pp));
        pp.qw = qweight;
        pp.bscale = block_scales;
        pp.tscale = tensor_scale;
        pp.Y = Y;
        pp.M = (int)M;
        pp.N = (int)N;
        pp.K = (int)K;
        pp.group_size = B;
        pp.G = (int)(K / B);
        pp.out_dtype = (int)out_dtype;
        pp.KA = (int)(K / 64);
        pp.tiles = (int)(N / 16);
        return format == W4_FP4_NVFP4 ? launch_prefill<false, w4p::kWNvfp4>(map, pp, dev, strm)
                                      : launch_prefill<false, w4p::kWMxfp4>(map, pp, dev, strm);
    }
    const size_t need = w4a16_fp4_workspace_bytes(M, N, K, format);
    if (need == 0) return W4_ERR_CUDA;
    if (!workspace || workspace_bytes < need) return W4_ERR_INVALID_ARG;
    w4d::DecodeParams p;
    std::memset(&p, 0, sizeof(p));
    p.qw = qweight;
    p.scales = reinterpret_cast<const __half*>(block_scales);
    p.tscale = tensor_scale;
    p.Y = Y;
    p.M = (int)M;
    p.N = (int)N;
    p.K = (int)K;
    p.group_size = B;
    p.G = (int)(K / B);
    p.out_dtype = (int)out_dtype;
    p.KA = (int)(K / 64);
    p.tiles = (int)(N / 16);
    const int mode = format == W4_FP4_NVFP4 ? w4d::kModeNvfp4 : w4d::kModeMxfp4;
    return dispatch_decode<false>(mode, p, X, reinterpret_cast<unsigned char*>(workspace),
                                  pre_offset(8, sm_count(dev)), dev, strm);
}
