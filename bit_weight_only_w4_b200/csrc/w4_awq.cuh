// w4_awq.cuh -- AWQ's per-channel scale search on a calibration batch.
//
// "Quantization Paradigms for Edge Inference: AWQ, GPTQ, and FP8 Matrix Cores", sec. 3:
// the salient channels are found from activation magnitudes under a calibration
// distribution, and s minimises L(s) = || W X - Q(W diag(s)) diag(s)^-1 X ||_2 (eq. 2).
// The candidates are the powers of the per-channel mean magnitude m[k] = mean_i |X[i,k]|:
//   s_a[k] = m[k]^a / geomean_k(m^a) = exp(a (log m[k] - mean_k log m)),  a = j / n_grid,
// each quantised by the library's quantiser and multiplied by its GEMM; these kernels add
// the magnitude statistics, the scale vector, the unquantised reference product and the
// loss.  Sums run in a fixed order, so the search is deterministic.
#pragma once
#include "w4_common.cuh"

namespace w4s {

template <bool BF16>
W4_DEV float load16(const void* p, size_t idx) {
    const unsigned short b = reinterpret_cast<const unsigned short*>(p)[idx];
    if constexpr (BF16) return __bfloat162float(__ushort_as_bfloat16(b));
    else return __half2float(__ushort_as_half(b));
}

// logm[k] = log(mean_i |X[i,k]|) in fp64, rows summed in order (a zero column gives
// log(1e-30)).
template <bool BF16>
__global__ void col_logmean_kernel(const void* __restrict__ X, int M, int K, double* __restrict__ logm) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    double s = 0.0;
    for (int i = 0; i < M; ++i) s += fabs((double)load16<BF16>(X, (size_t)i * K + k));
    logm[k] = log(fmax(s / M, 1e-30));
}

// mu = mean_k logm[k] (fp64, channels in order; one thread).
__global__ void mean_kernel(const double* __restrict__ v, int K, double* __restrict__ mu) {
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    double s = 0.0;
    for (int k = 0; k < K; ++k) s += v[k];
    *mu = s / K;
}

// s[k] = fp32(exp(a (logm[k] - mu))), s_inv[k] = 1 / s[k] (one fp32 division).
__global__ void awq_scale_kernel(const double* __restrict__ logm, const double* __restrict__ mu, double a,
                                 int K, float* __restrict__ s, float* __restrict__ s_inv) {
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    const float v = (float)exp(a * (logm[k] - *mu));
    s[k] = v;
    s_inv[k] = __fdiv_rn(1.0f, v);
}

// Y[i,n] = sum_k X[i,k] W[n,k] with fp32 products and sums (k ascending in 16-wide tiles),
// 16 x 16 outputs per block.
constexpr int kT = 16;
template <bool XBF16, bool WBF16>
__global__ void ref_gemm_kernel(const void* __restrict__ X, const void* __restrict__ W, int M, int N, int K,
                                float* __restrict__ Y) {
    __shared__ float xs[kT][kT + 1], ws[kT][kT + 1];
    const int tx = threadIdx.x, ty = threadIdx.y;
    const int i = blockIdx.y * kT + ty, n = blockIdx.x * kT + tx;
    float acc = 0.0f;
    for (int k0 = 0; k0 < K; k0 += kT) {
        const int i_l = blockIdx.y * kT + ty, k_l = k0 + tx;
        xs[ty][tx] = (i_l < M && k_l < K) ? load16<XBF16>(X, (size_t)i_l * K + k_l) : 0.0f;
        const int n_l = blockIdx.x * kT + ty;
        ws[ty][tx] = (n_l < N && k_l < K) ? load16<WBF16>(W, (size_t)n_l * K + k_l) : 0.0f;
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < kT; ++kk) acc = __fmaf_rn(xs[ty][kk], ws[tx][kk], acc);
        __syncthreads();
    }
    if (i < M && n < N) Y[(size_t)i * N + n] = acc;
}

// partial[b] = sum over elements [b * chunk, (b + 1) * chunk) of (A - B)^2 in fp64, each
// block reducing in a fixed tree order.
constexpr int kLossThreads = 256;
__global__ void sqdiff_partial_kernel(const float* __restrict__ A, const float* __restrict__ B, size_t n,
                                      size_t chunk, double* __restrict__ partial) {
    __shared__ double red[kLossThreads];
    const size_t lo = (size_t)blockIdx.x * chunk, hi = min(n, lo + chunk);
    double s = 0.0;
    for (size_t i = lo + threadIdx.x; i < hi; i += kLossThreads) {
        const double d = (double)A[i] - (double)B[i];
        s += d * d;
    }
    red[threadIdx.x] = s;
    __syncthreads();
    for (int w = kLossThreads / 2; w > 0; w >>= 1) {
        if (threadIdx.x < w) red[threadIdx.x] += red[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) partial[blockIdx.x] = red[0];
}

// out = sum_b partial[b] in order (one thread).
__global__ void sum_kernel(const double* __restrict__ partial, int nb, double* __restrict__ out) {
    if (blockIdx.x != 0 || threadIdx.x != 0) return;
    double s = 0.0;
    for (int b = 0; b < nb; ++b) s += partial[b];
    *out = s;
}

}  // namespace w4s
