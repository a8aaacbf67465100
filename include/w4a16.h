/*
 * w4a16.h -- C ABI of the B200 (sm_100a) W4A16 library: 4-bit weight-only quantised
 * linear layers with 16-bit activations.
 *
 * The method (page title, section):
 *  - AWQ equivalence transform: "Quantization Paradigms for Edge Inference: AWQ, GPTQ,
 *    and FP8 Matrix Cores", sec. 3 "The Math Behind Activation-Aware Protection (AWQ)",
 *    eq. 1: W' = W diag(s), X' = diag(s)^-1 X, so W'X' = WX.  Salient input channels
 *    are scaled up in the weights and down in the activations instead of being kept in
 *    fp16 (edgesiliconlab.com article on AWQ vs GPTQ, "What Is the Core Difference
 *    Between AWQ and GPTQ Quantization?").
 *  - Group-wise asymmetric round-to-nearest INT4 with per-group scales and zero points:
 *    "The Ultimate Guide to Quantized LLMs: GPTQ", "Understanding Quantized Model
 *    Compression"; edgesiliconlab.com article, "Quantization on Non-NVIDIA Silicon".
 *  - Two 4-bit weights per byte, unpacked with shift/AND to 16-bit just before the
 *    tensor cores, with staged, double-buffered weight tiles: edgesiliconlab.com
 *    article, "Kernel Execution: Marlin vs. ExLlamaV2 INT4 GEMM Micro-Architecture",
 *    items 1-3.  Decode reads every weight once and is bandwidth-bound, prefill is
 *    compute-bound: same article, "The Mathematics of Memory Bandwidth Saturation".
 *
 * Conventions shared by every entry point
 *  - All pointers named as "device" are CUDA device (or managed) pointers of the
 *    current device; the caller owns every buffer and keeps it alive until the work
 *    on `stream` has finished.  The library never allocates device memory.
 *  - Calls are asynchronous and stream-ordered on `stream` (NULL = legacy default
 *    stream).  Arguments are validated on the host before any launch; the returned
 *    status is synchronous.  W4_ERR_CUDA means a launch failed (cudaGetLastError).
 *  - Kernels never trap.  Every wait inside a kernel is bounded; on expiry the kernel
 *    records a device-side error word and returns.  w4_check_device_error() reads it.
 *  - No C++ exception crosses this ABI.  The library keeps no per-call host state, so
 *    calls from several host threads on different streams are safe.
 *  - Shapes: N % 16 == 0, N <= 1048576, K % 64 == 0, group_size == 32 or a multiple
 *    of 64, and K % group_size == 0 (group_size == K is per-channel).  Pointers to packed weights,
 *    activations, outputs and fp16 metadata must be 16-byte aligned.
 *
 * Packed weight format ("device layout")
 *  The INT4 codes q[n][k] in [0,15] of W [N,K] are stored as N*K/8 uint32 words in
 *  atoms of 16 rows x 64 columns (128 words).  Eight consecutive row tiles form a band of
 *  128 rows (the last band holds Tb = min(8, N/16 - 8b) tiles).  Band b starts at atom
 *  8*(K/64)*b; inside it the atom of row tile tt (rows 16(8b+tt)..+15) and column block a
 *  (columns 64a..64a+63) is atom a*Tb + tt, i.e. a band is stored column block by column
 *  block, so consecutive column blocks of a band are one contiguous run.  Word 4L+j of an
 *  atom (L = 0..31, j = 0..3) holds, with t = 8b+tt, r0 = 16t + L/4, r1 = r0 + 8,
 *  kb = 64a + 16j, c = 2*(L%4), nibble i in bits 4i..4i+3:
 *     nibble 0: q[r0][kb+c]     nibble 4: q[r0][kb+c+1]
 *     nibble 1: q[r1][kb+c]     nibble 5: q[r1][kb+c+1]
 *     nibble 2: q[r0][kb+c+8]   nibble 6: q[r0][kb+c+9]
 *     nibble 3: q[r1][kb+c+8]   nibble 7: q[r1][kb+c+9]
 *  Lane L of a warp loads words 4L..4L+3 of an atom with one 16-byte load; each word is
 *  then exactly the 16x16 weight operand slice that lane needs for one 16-deep step of
 *  a warp-level MMA, and the eight codes come out as fp16/bf16 pairs with one
 *  AND/OR per pair (the exponent-bias trick) plus one subtract.
 *  The "canonical layout" (w4_unpack_canonical) is uint32 [N, K/8] with nibble j of
 *  word i of row n equal to q[n][8i+j].
 *
 *  scales: fp16 [G, N] (G = K/group_size), scale of group g of output row n at
 *          scales[g*N + n].  zeros: fp16 [G, N] holding the integer zero point z in
 *          [0,15]; NULL means the symmetric format with implicit z = 8.
 *  Dequantised weight: (q - z) * scale.
 */
#ifndef W4A16_H
#define W4A16_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st* w4_stream_t;

typedef enum {
    W4_OK = 0,
    W4_ERR_INVALID_ARG = 1, /* NULL / misaligned pointer, negative or inconsistent size */
    W4_ERR_UNSUPPORTED = 2, /* legal but not tiled: see the shape rules above          */
    W4_ERR_CUDA = 3,        /* a CUDA call or kernel launch failed                      */
    W4_ERR_TIMEOUT = 4,     /* a kernel gave up a bounded wait (device error word)      */
    W4_ERR_DEVICE_ARG = 5   /* a kernel found an out-of-range g_idx entry               */
} w4_status;

typedef enum { W4_F16 = 0, W4_BF16 = 1, W4_F32 = 2 } w4_dtype;

/*
 * w4_quantize_pack -- AWQ weight scaling + group-wise RTN INT4 + packing.
 *
 * Computes, for every output row n and group g (channels k with group(k) == g, where
 * group(k) = g_idx[k] if g_idx != NULL else k / group_size):
 *   W'[n,k] = float(W[n,k]) * s[k]                  (fp32, one rounding; s NULL = 1)
 *   asymmetric: sc = fp16(max((max W' - min W')/15, 2^-14)),
 *               z  = clamp(rint(-min W' / sc), 0, 15)           (stored as fp16 z)
 *   symmetric:  sc = fp16(max(max|W'| / 7, 2^-14)), z = 8        (not stored)
 *   q[n,k] = clamp(rint(W'[n,k] / sc) + z, 0, 15)   (IEEE fp32 division, rint =
 *                                                    round half to even)
 * and packs q into the device layout above.  Bit-exact: no fast-math anywhere.
 *
 *   W          device, [N,K] row-major, fp16 (w_dtype W4_F16) or bf16 (W4_BF16)
 *   s          device fp32 [K] AWQ per-input-channel scale, or NULL
 *   group_size 32 or a multiple of 64, K % group_size == 0
 *   symmetric  0 = asymmetric (zeros required), 1 = symmetric (zeros must be NULL)
 *   g_idx      device int32 [K] group of each input channel (act-order), or NULL;
 *              entries outside [0, K/group_size) are skipped and reported as
 *              W4_ERR_DEVICE_ARG by w4_check_device_error()
 *   qweight    device uint32 [N*K/8] output, device layout
 *   scales     device fp16 [G,N] output;  zeros device fp16 [G,N] output or NULL
 * Uses 128*G bytes of shared memory per tile of 16 rows (G = K/group_size):
 * K/group_size above 1536 returns W4_ERR_UNSUPPORTED.
 */
w4_status w4_quantize_pack(const void* W, w4_dtype w_dtype, int64_t N, int64_t K,
                           const float* s, int32_t group_size, int32_t symmetric,
                           const int32_t* g_idx, uint32_t* qweight, void* scales,
                           void* zeros, w4_stream_t stream);

/*
 * w4a16_gemm -- fused dequantise-GEMM:  Y[M,N] = X'[M,K] * What[N,K]^T, with
 *   X'[m,k]   = X[m,k] * s_inv[k]   (s_inv NULL: X' = X)   -- AWQ eq. 1, right factor
 *   What[n,k] = (q[n,k] - z[group(k),n]) * scale[group(k),n]
 * accumulated in fp32.  Without g_idx the codes reach the tensor cores as exact small
 * integers and each group's fp32 partial sum is multiplied by its scale: the prefill
 * kernel multiplies (q - z); the decode kernel multiplies the biased codes the AND/OR
 * unpack yields (1024 + q or 1024 + 16 q in fp16, 128 + q in bf16) and removes the bias
 * and the zero point per group with the group's activation sum, in fp32.  With g_idx the
 * scale is folded into an fp16 weight before the MMA (fp16 activations only).  With
 * s_inv, X' is rounded to the activation dtype before the MMA.
 *
 *   X          device [M,K] row-major, act_dtype W4_F16 or W4_BF16
 *   qweight, scales, zeros, g_idx, group_size: as produced by w4_quantize_pack
 *   s_inv      device fp32 [K] or NULL
 *   Y          device [M,N] row-major output, out_dtype W4_F16, W4_BF16 or W4_F32
 *   workspace  device scratch of at least w4a16_workspace_bytes(M,N,K,group_size)
 *              bytes, 256-byte aligned, ZERO-FILLED BEFORE ITS FIRST USE;
 *              every call leaves it zero-filled again where that matters, so one
 *              workspace may be reused by any number of calls on one stream.  Calls
 *              that may overlap on the GPU need separate workspaces.  After a call
 *              whose kernel reported W4_ERR_TIMEOUT, zero it again.
 * M == 0 is a no-op.  M <= 64 runs the bandwidth-bound decode kernel (warp MMAs,
 * split-K across the GPU), larger M the tcgen05 tensor-core kernel.
 * bf16 activations with g_idx return W4_ERR_UNSUPPORTED.
 */
w4_status w4a16_gemm(const void* X, w4_dtype act_dtype, int64_t M, int64_t N, int64_t K,
                     const uint32_t* qweight, const void* scales, const void* zeros,
                     const int32_t* g_idx, int32_t group_size, const float* s_inv,
                     void* Y, w4_dtype out_dtype, void* workspace, size_t workspace_bytes,
                     w4_stream_t stream);

/*
 * Act-order weights with contiguous groups.  An act-order vector g_idx scatters each
 * group's channels along K ("The Ultimate Guide to Quantized LLMs: GPTQ" and
 * "Understanding Quantized Model Compression": one scale and zero point per group of
 * input channels).  When every group holds exactly group_size channels, ordering the
 * channels by group makes each group a contiguous run again, and the product is the same
 * sum taken in that order:
 *   perm[k'] = the k'-th channel in (g_idx[k], k) order   (a stable sort by group)
 *   Y[m,n]   = sum_k' X'[m,perm[k']] * What[n,perm[k']],  group(perm[k']) = k' / group_size.
 * w4_quantize_pack_perm packs column k' = channel perm[k'] (codes, scales and zero points
 * identical to w4_quantize_pack with g_idx, the codes in k' order); w4a16_gemm_perm gathers
 * the activation columns through perm (with s_inv of the original channel) and runs the
 * contiguous-group kernels, so act-order weights stream at the speed of ordinary ones.
 */

/*
 * w4_actorder_perm -- perm = the channels sorted by g_idx, ties in channel order.
 *   g_idx      device int32 [K], every entry in [0, K/group_size)
 *   perm       device int32 [K] output, 16-byte aligned
 * One warp walks K in order (offline, once per layer).  Every group must hold exactly
 * group_size channels: otherwise, or for an entry outside [0, K/group_size), perm is
 * incomplete and w4_check_device_error() reports W4_ERR_DEVICE_ARG.  More than 12288 groups
 * return W4_ERR_UNSUPPORTED.
 */
w4_status w4_actorder_perm(const int32_t* g_idx, int64_t K, int32_t group_size, int32_t* perm,
                           w4_stream_t stream);

/*
 * w4_quantize_pack_perm -- w4_quantize_pack of the column-permuted matrix: column k of the
 * packed result is channel perm[k] of W (and of s); groups are k / group_size.  Arguments
 * as w4_quantize_pack, with perm (device int32 [K], entries in [0, K)) in place of g_idx.
 * An entry outside [0, K) reads channel 0 and is reported as W4_ERR_DEVICE_ARG by
 * w4_check_device_error().
 */
w4_status w4_quantize_pack_perm(const void* W, w4_dtype w_dtype, int64_t N, int64_t K,
                                const float* s, int32_t group_size, int32_t symmetric,
                                const int32_t* perm, uint32_t* qweight, void* scales,
                                void* zeros, w4_stream_t stream);

/*
 * w4a16_gemm_perm -- Y = X' What^T for weights packed by w4_quantize_pack_perm:
 *   Xp[m,k'] = X[m,perm[k']] * s_inv[perm[k']]  rounded to act_dtype (s_inv NULL: no scaling).
 * When the decode kernel keeps X' resident in shared memory (M <= 8 and M*K small), it
 * gathers the columns itself while preparing X', in the one launch.  Otherwise one gather
 * kernel writes Xp into the workspace and w4a16_gemm(Xp, ..., g_idx = NULL, s_inv = NULL)
 * follows.  Arguments as w4a16_gemm with perm in place of g_idx; fp16 and bf16
 * activations.  workspace: at least w4a16_workspace_bytes_perm(M,N,K,group_size) bytes,
 * 256-byte aligned, zero-filled before its first use (as for w4a16_gemm).  An entry of perm
 * outside [0, K) reads channel 0 and is reported as W4_ERR_DEVICE_ARG by
 * w4_check_device_error().
 */
w4_status w4a16_gemm_perm(const void* X, w4_dtype act_dtype, int64_t M, int64_t N, int64_t K,
                          const uint32_t* qweight, const void* scales, const void* zeros,
                          const int32_t* perm, int32_t group_size, const float* s_inv,
                          void* Y, w4_dtype out_dtype, void* workspace, size_t workspace_bytes,
                          w4_stream_t stream);

/* Bytes of workspace w4a16_gemm_perm needs (w4a16_workspace_bytes plus M*K*2 for the
 * gathered activations; 0 on invalid sizes). */
size_t w4a16_workspace_bytes_perm(int64_t M, int64_t N, int64_t K, int32_t group_size);

/*
 * w4_awq_search -- AWQ's per-channel scale search on a calibration batch ("Quantization
 * Paradigms for Edge Inference: AWQ, GPTQ, and FP8 Matrix Cores", sec. 3: s minimises
 * L(s) = || W X - Q(W diag(s)) diag(s)^-1 X ||_2, found from activation magnitudes).
 * Candidates: with m[k] = mean_i |X[i,k]| and a_j = j / n_grid (j = 0 .. n_grid-1),
 *   s_j[k] = fp32(exp(a_j (log m[k] - mean_k log m)))     (m^a_j over its geometric mean;
 *                                                          s_0 = 1, plain RTN),
 *   L_j    = sum_{i,n} (Yref[i,n] - Yq_j[i,n])^2          (fp64 sum of fp32 terms),
 * with Yref = X W^T in fp32 and Yq_j = w4a16_gemm(X, w4_quantize_pack(W, s_j), s_inv =
 * 1/s_j) in fp32.  Returns the first j of the smallest L_j.
 *
 *   W          device [N,K] row-major fp16/bf16 (w_dtype); X device [M,K] calibration rows
 *              (x_dtype); 1 <= M <= 2^19; group_size, symmetric as for w4_quantize_pack
 *   n_grid     1..1024 candidates
 *   s_best     device fp32 [K] output: the chosen s (pass it to w4_quantize_pack, and its
 *              reciprocal as the GEMM's s_inv)
 *   losses     HOST fp64 [n_grid] output: L_j
 *   best       HOST int32 output: the chosen j
 *   workspace  device scratch of w4_awq_search_workspace_bytes(...) bytes, 256-byte
 *              aligned, zero-filled before its first use (it holds a w4a16_gemm workspace)
 * Offline and synchronous: the call waits for the stream before it returns.  Device-side
 * errors of the kernels it runs are reported by w4_check_device_error().
 */
w4_status w4_awq_search(const void* W, w4_dtype w_dtype, int64_t N, int64_t K, const void* X,
                        w4_dtype x_dtype, int64_t M, int32_t group_size, int32_t symmetric,
                        int32_t n_grid, float* s_best, double* losses, int32_t* best,
                        void* workspace, size_t workspace_bytes, w4_stream_t stream);

/* Bytes of workspace w4_awq_search needs (0 on invalid sizes). */
size_t w4_awq_search_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t group_size,
                                     int32_t symmetric, int32_t n_grid);

/*
 * w4a16_gemm_chain -- a list of small-batch GEMMs in order, in one persistent launch per
 * 32 layers: Y_l = (X_l * s_inv_l) @ dequant(W_l)^T for l = 0, 1, ..., each exactly as
 * w4a16_gemm computes it for the same M.  A decode step reads every weight once per
 * token and is bound by memory bandwidth (edgesiliconlab.com article on AWQ vs GPTQ,
 * "The Mathematics of Memory Bandwidth Saturation"); in one launch the packed weights
 * of layer l+1 are already streaming while the GPU finishes layer l, which separate
 * launches cannot do.
 *
 * Layer l+1 starts reading X_{l+1} only after every output of layers 0..l is stored, so
 * X_{l+1} may point into the output of any earlier layer of the list (a slice of a row:
 * X + offset with row stride ldx).  Each X_l row holds K_l values of act_dtype; Y_l is
 * written in out_dtype, so a layer that feeds a later one wants out_dtype == act_dtype.
 *
 *   layers     HOST array of n_layers descriptors (read during the call only):
 *                X       device [M, K] activations, rows ldx elements apart
 *                        (ldx >= K, ldx % 8 == 0), 16-byte aligned
 *                qweight, scales, zeros, group_size, N, K: as for w4a16_gemm (no g_idx)
 *                s_inv   device fp32 [K] or NULL
 *                Y       device [M, N] output (row-major, rows N apart)
 *   M          1..8; every layer's M*K*2 bytes of X' plus its channel sums must fit the
 *              resident budget (120 KB, leaving the weight ring at least three stages),
 *              else W4_ERR_UNSUPPORTED (K = 11008 allows M <= 4, K = 4096 every M <= 8)
 *   every layer must use the same group handling: group sizes all multiples of 128 with
 *              K % 128 == 0, or all 32, or all other multiples of 64
 *   workspace  device, >= w4a16_chain_workspace_bytes(M) bytes, 256-byte aligned,
 *              ZERO-FILLED BEFORE ITS FIRST USE; each launch leaves it zero again (a
 *              w4a16_gemm workspace of at least this size may be shared with it on one
 *              stream); after W4_ERR_TIMEOUT zero it again
 * All CTAs of a launch (one per SM) must be resident together, which holds when no
 * other work occupies the GPU's SMs; the waits between layers are bounded and report
 * W4_ERR_TIMEOUT through w4_check_device_error() if that is ever violated.
 * Asynchronous on `stream`.  n_layers == 0 or M == 0 is a no-op.
 */
typedef struct {
    const void* X;
    int64_t ldx;
    const uint32_t* qweight;
    const void* scales;
    const void* zeros;
    const float* s_inv;
    void* Y;
    int64_t N;
    int64_t K;
    int32_t group_size;
} w4_chain_layer;

w4_status w4a16_gemm_chain(const w4_chain_layer* layers, int32_t n_layers, int64_t M,
                           w4_dtype act_dtype, w4_dtype out_dtype, void* workspace,
                           size_t workspace_bytes, w4_stream_t stream);

/* Bytes of workspace w4a16_gemm_chain needs on the current device (0 unless 1 <= M <= 8). */
size_t w4a16_chain_workspace_bytes(int64_t M);

/*
 * Block-scaled 4-bit floating-point weights (NVFP4, MXFP4), the Blackwell 4-bit format
 * of "Production Quantization: AWQ, GPTQ, GGUF K-quants, FP8, MXFP4/NVFP4", section
 * "MXFP4 / NVFP4" (4-bit floating-point values with a scale per block of weights): a
 * comparator for the INT4 path on the same layer shapes, with 16-bit activations.
 *   element  E2M1: sign, 2 exponent bits, 1 mantissa bit; magnitudes 0, 0.5, 1, 1.5,
 *            2, 3, 4, 6
 *   NVFP4    blocks of 16 consecutive input channels, an E4M3 block scale sb, one fp32
 *            tensor scale gs = amax|W| / (6 * 448) (1 for an all-zero W):
 *            sb = E4M3(blockmax / 6 / gs), q = E2M1(w / (E4M3(sb) * gs))
 *   MXFP4    blocks of 32, a power-of-two scale 2^e stored as the byte e + 127,
 *            e = max(floor(log2 blockmax) - 2, -127), q = E2M1(w / 2^e)
 * All in fp32; every conversion rounds to nearest, ties to even, and saturates finite
 * values at the largest magnitude; an element's sign is its input's, also at zero.
 */
typedef enum { W4_FP4_NVFP4 = 0, W4_FP4_MXFP4 = 1 } w4_fp4_format;

/*
 * w4_fp4_quantize_pack -- quantise W to NVFP4 or MXFP4 and pack the codes.
 *   W             device [N,K] row-major, fp16 (W4_F16) or bf16 (W4_BF16)
 *   N, K          N % 16 == 0, K % 64 == 0
 *   qweight       device uint32 [N*K/8] output: the E2M1 codes in the device layout of
 *                 the INT4 codes above (code (n,k) where q[n][k] would be)
 *   block_scales  device uint8 [K/B, N] output (B = 16 NVFP4, 32 MXFP4), block-row-major
 *   tensor_scale  device fp32 [1] output for NVFP4 (gs); must be NULL for MXFP4
 * Bit-exact (no fast-math).  Asynchronous on `stream`.
 */
w4_status w4_fp4_quantize_pack(const void* W, w4_dtype w_dtype, int64_t N, int64_t K,
                               w4_fp4_format format, uint32_t* qweight, uint8_t* block_scales,
                               float* tensor_scale, w4_stream_t stream);

/*
 * w4a16_fp4_gemm -- Y[M,N] = X[M,K] @ What^T, What[n,k] = E2M1(q[n,k]) * scale(block of
 * k, n) (* gs for NVFP4), fp32 accumulation.  fp16 activations only (every E2M1 value is
 * exact in fp16; bf16 returns W4_ERR_UNSUPPORTED).  M <= 64 runs the bandwidth-bound
 * decode kernel: each block's products are summed by the tensor cores and multiplied by
 * the block's scale (times gs) in fp32.  Larger M runs the tcgen05 prefill kernel on
 * weights decoded to fp16 with their block scale (E2M1 x E4M3 and E2M1 x 2^e are exact in
 * fp16 for e in [-13, 13]), the whole K accumulating in tensor memory and gs applied at
 * the end; an MXFP4 block whose e lies outside [-13, 13] (other than the byte 0, whose
 * block reads as zero) is reported as W4_ERR_DEVICE_ARG by w4_check_device_error().
 *   workspace  >= w4a16_fp4_workspace_bytes(M,N,K,format) bytes, 256-byte aligned,
 *              zero-filled before its first use (as for w4a16_gemm)
 */
w4_status w4a16_fp4_gemm(const void* X, w4_dtype act_dtype, int64_t M, int64_t N, int64_t K,
                         const uint32_t* qweight, const uint8_t* block_scales,
                         const float* tensor_scale, w4_fp4_format format, void* Y,
                         w4_dtype out_dtype, void* workspace, size_t workspace_bytes,
                         w4_stream_t stream);

/* Bytes of workspace w4a16_fp4_gemm needs (0 on invalid sizes, and for M > 64, which
 * needs none). */
size_t w4a16_fp4_workspace_bytes(int64_t M, int64_t N, int64_t K, w4_fp4_format format);

/*
 * w4a16_gemm_noalloc -- w4a16_gemm for 1 <= M <= 32 without a caller-supplied
 * workspace.  The pages have no counterpart to this call; it
 * exists for callers that cannot allocate device memory where they run the GEMM, such as
 * plug-ins of inference runtimes that forbid allocation after their set-up phase, or C
 * callers without a caching allocator, for whom cudaMalloc/cudaFree per call would
 * synchronise the whole device.
 *
 * Arguments, layouts and results are those of w4a16_gemm minus the workspace.  The
 * scratch is one fixed 8 MiB array in device memory that every GPU loading this library
 * holds until the process exits: the split-K slots of up to four token tiles, then the
 * prepared activations (M*K*2 bytes plus their sums, K up to about 48000 at M = 32 on a
 * 148-SM B200).  Calls beyond it (M > 32, or a larger M*K) return W4_ERR_UNSUPPORTED;
 * use w4a16_gemm for them.  The
 * first call on a device sets up that device (looks up the array's address, zeroes the
 * array and synchronises the device); make that first call before any stream
 * capture.  If the set-up fails the call returns W4_ERR_CUDA and the next call tries it
 * again.  Every call on a device shares the one array: calls that may overlap on the
 * GPU (different streams without ordering) race and give wrong results.  A call whose
 * kernel gave up a bounded wait can leave split-K flags set in the array; when
 * w4_check_device_error() reports W4_ERR_TIMEOUT it zeroes the array of the current
 * device again, so later calls start clean.  The call allocates nothing and frees
 * nothing.
 */
w4_status w4a16_gemm_noalloc(const void* X, w4_dtype act_dtype, int64_t M, int64_t N, int64_t K,
                             const uint32_t* qweight, const void* scales, const void* zeros,
                             const int32_t* g_idx, int32_t group_size, const float* s_inv,
                             void* Y, w4_dtype out_dtype, w4_stream_t stream);

/* Bytes of workspace w4a16_gemm needs for these sizes on the current device
 * (0 on invalid sizes). */
size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K, int32_t group_size);

/* Test aid: convert device-layout packed weights to the canonical layout
 * (uint32 [N, K/8], nibble j of word i of row n = q[n][8i+j]).  Both device pointers. */
w4_status w4_unpack_canonical(const uint32_t* qweight, int64_t N, int64_t K,
                              uint32_t* qweight_canonical, w4_stream_t stream);

/* Synchronises the current device, then reports and clears the device-side error word:
 * W4_ERR_TIMEOUT if a kernel gave up a bounded wait, W4_ERR_DEVICE_ARG if a kernel met
 * an out-of-range g_idx or permutation entry or an MXFP4 block scale the prefill kernel
 * cannot decode exactly, W4_ERR_CUDA if the device reports a CUDA error, W4_OK.
 * On W4_ERR_TIMEOUT it also zeroes the current device's w4a16_gemm_noalloc scratch again
 * (a timed-out kernel may have left split-K flags in it); workspaces passed to
 * w4a16_gemm belong to the caller, who zeroes them again. */
w4_status w4_check_device_error(void);

/* Bound, in nanoseconds, of every wait inside the library's kernels (default 2e9).
 * Lowering it is a test aid; values below 1000 are raised to 1000. */
w4_status w4_set_wait_limit_ns(uint64_t ns);

/* Test aid for the watchdog: launches one block whose thread waits on a barrier that
 * nothing completes; the bounded wait expires after the configured limit and sets the
 * device error word (so w4_check_device_error() then returns W4_ERR_TIMEOUT). */
w4_status w4_selftest_expired_wait(w4_stream_t stream);

/* Test aid for w4a16_gemm_noalloc's recovery, on the current device (synchronous).
 * plant != 0: sets every split-K word of the allocation-free scratch to a flagged stale
 * partial (what a kernel that gave up a wait can leave behind); *nonzero_words, if not
 * NULL, receives the number of words written.  plant == 0: counts the scratch's nonzero
 * split-K words into *nonzero_words (0 once w4_check_device_error() has zeroed it). */
w4_status w4_selftest_noalloc_scratch(int32_t plant, uint64_t* nonzero_words);

/* Static string naming a status. */
const char* w4_status_string(w4_status status);

#ifdef __cplusplus
}
#endif

#endif /* W4A16_H */
