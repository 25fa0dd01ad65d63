// w4_awq_search: the AWQ smoothing-scale search on the GPU.
//
// Method: page 2 (learn.longtimenohack.com/chasing/pages/quantization.html),
// AWQ section, the awq_search_scale listing: act = the mean magnitude of each
// input channel over the calibration rows; for alpha on an even grid over
// [0, 1], s = act^alpha / mean(act^alpha); quantize and dequantize W * s; the
// loss is mean((W X^T - (W^ / s) X^T)^2); keep the alpha with the smallest
// loss.  The exact readings are stated in include/w4.h.
//
// Every step runs in this library's kernels: the channel magnitudes and the
// reference product W X^T once per search (fp32 accumulation of the bf16
// inputs), then per alpha the scale vector, w4_quant_pack with the fold, the
// activations divided by s, w4a16_gemm on them (the product (W^/s) X^T as the
// W4A16 path computes it) and a squared-error reduction in fp64.  All work is
// enqueued on the caller's stream; the scratch is the caller's workspace.
#include "common.cuh"

#include <algorithm>

namespace w4 {
namespace {

__global__ void act_kernel(const __nv_bfloat16 *__restrict__ X, int M, int K, double *__restrict__ act)
{
    const int k = blockIdx.x * blockDim.x + threadIdx.x;
    if (k >= K) return;
    double s = 0.0;
    for (int m = 0; m < M; ++m) s += fabs((double)__bfloat162float(X[(size_t)m * K + k]));
    act[k] = s / (double)M;
}

// s[k] = fl32(act[k]^alpha / mean_k act^alpha), alpha = ia / (n_alpha - 1);
// one CTA of 1024 threads.  With best != nullptr the index is read from it.
__global__ void __launch_bounds__(1024) scale_kernel(const double *__restrict__ act, int K, int ia, const int *best,
                                                     int n_alpha, float *__restrict__ s)
{
    __shared__ double red[32];
    const int i = best ? *best : ia;
    const double alpha = (double)i / (double)(n_alpha - 1);
    double sum = 0.0;
    for (int k = threadIdx.x; k < K; k += blockDim.x) sum += pow(act[k], alpha);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = sum;
    __syncthreads();
    if (threadIdx.x < 32) {
        double v = threadIdx.x < (blockDim.x >> 5) ? red[threadIdx.x] : 0.0;
#pragma unroll
        for (int off = 16; off > 0; off >>= 1) v += __shfl_xor_sync(0xffffffffu, v, off);
        if (threadIdx.x == 0) red[0] = v;
    }
    __syncthreads();
    const double mean = red[0] / (double)K;
    for (int k = threadIdx.x; k < K; k += blockDim.x) s[k] = (float)(pow(act[k], alpha) / mean);
}

// Xs = bf16(fl32(x) / s[k]) (IEEE division)
__global__ void xdiv_kernel(const __nv_bfloat16 *__restrict__ X, const float *__restrict__ s, int64_t MK, int K,
                            __nv_bfloat16 *__restrict__ Xs)
{
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < MK; i += (int64_t)gridDim.x * blockDim.x)
        Xs[i] = __float2bfloat16_rn(__fdiv_rn(__bfloat162float(X[i]), s[i % K]));
}

// Y[m][n] = sum_k x[m][k] * w[n][k], fp32 accumulation: 64 x 64 outputs per CTA,
// 4 x 4 per thread, 32-wide k-slices staged in shared memory.
__global__ void __launch_bounds__(256) ref_gemm_kernel(const __nv_bfloat16 *__restrict__ X,
                                                       const __nv_bfloat16 *__restrict__ W, int M, int N, int K,
                                                       float *__restrict__ Y)
{
    __shared__ float xs[32][65], ws[32][65];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    float acc[4][4] = {};
    for (int k0 = 0; k0 < K; k0 += 32) {
        for (int e = threadIdx.x; e < 64 * 32; e += 256) {
            const int r = e >> 5, kk = e & 31;
            const int m = m0 + r, n = n0 + r, k = k0 + kk;
            xs[kk][r] = (m < M && k < K) ? __bfloat162float(X[(size_t)m * K + k]) : 0.f;
            ws[kk][r] = (n < N && k < K) ? __bfloat162float(W[(size_t)n * K + k]) : 0.f;
        }
        __syncthreads();
#pragma unroll 8
        for (int kk = 0; kk < 32; ++kk) {
            float a[4], b[4];
#pragma unroll
            for (int u = 0; u < 4; ++u) {
                a[u] = xs[kk][ty + 16 * u];
                b[u] = ws[kk][tx + 16 * u];
            }
#pragma unroll
            for (int u = 0; u < 4; ++u)
#pragma unroll
                for (int v = 0; v < 4; ++v) acc[u][v] = fmaf(a[u], b[v], acc[u][v]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int m = m0 + ty + 16 * u, n = n0 + tx + 16 * v;
            if (m < M && n < N) Y[(size_t)m * N + n] = acc[u][v];
        }
}

// acc += sum (Yref - Yq)^2 over all outputs, in fp64
__global__ void __launch_bounds__(256) sqerr_kernel(const float *__restrict__ Yref,
                                                    const __nv_bfloat16 *__restrict__ Yq, int64_t count,
                                                    double *__restrict__ acc)
{
    __shared__ double red[8];
    double local = 0.0;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < count; i += (int64_t)gridDim.x * blockDim.x) {
        const double d = (double)Yref[i] - (double)__bfloat162float(Yq[i]);
        local += d * d;
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) local += __shfl_xor_sync(0xffffffffu, local, off);
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = local;
    __syncthreads();
    if (threadIdx.x == 0) {
        double t = 0.0;
        for (int w = 0; w < 8; ++w) t += red[w];
        atomicAdd(acc, t);
    }
}

// losses[i] /= count; best = the first index of the minimum
__global__ void finish_kernel(double *losses, int n_alpha, double count, int *best)
{
    if (threadIdx.x != 0 || blockIdx.x != 0) return;
    int b = 0;
    for (int i = 0; i < n_alpha; ++i) {
        losses[i] /= count;
        if (losses[i] < losses[b]) b = i;
    }
    *best = b;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct AwqLayout {
    size_t act, s, xs, q, sc, z, yref, yq, gws, total;
};

AwqLayout awq_layout(int64_t M, int64_t N, int64_t K, int group, int mode)
{
    AwqLayout L;
    const int64_t G = K / group;
    size_t o = 0;
    L.act = o; o += align256((size_t)K * 8);
    L.s = o; o += align256((size_t)K * 4);
    L.xs = o; o += align256((size_t)M * K * 2);
    L.q = o; o += align256((size_t)N * K / 2);
    L.sc = o; o += align256((size_t)N * G * 2);
    L.z = o; o += (mode == W4_ASYM) ? align256((size_t)N * ((G + 7) / 8) * 4) : 0;
    L.yref = o; o += align256((size_t)M * N * 4);
    L.yq = o; o += align256((size_t)M * N * 2);
    L.gws = o; o += align256(w4a16_workspace_bytes(M, N, K, group));
    L.total = o;
    return L;
}

}  // namespace

size_t awq_workspace_bytes(int64_t M, int64_t N, int64_t K, int group, int mode)
{
    return awq_layout(M, N, K, group, mode).total;
}

cudaError_t launch_awq_search(const void *W, const void *X, int64_t N, int64_t K, int64_t M, int group, int mode,
                              int n_alpha, double *losses, int *best, float *s_best, void *ws, cudaStream_t stream)
{
    const AwqLayout L = awq_layout(M, N, K, group, mode);
    uint8_t *base = (uint8_t *)ws;
    double *act = (double *)(base + L.act);
    float *s = (float *)(base + L.s);
    __nv_bfloat16 *xs = (__nv_bfloat16 *)(base + L.xs);
    uint32_t *q = (uint32_t *)(base + L.q);
    void *sc = base + L.sc;
    uint32_t *z = mode == W4_ASYM ? (uint32_t *)(base + L.z) : nullptr;
    float *yref = (float *)(base + L.yref);
    __nv_bfloat16 *yq = (__nv_bfloat16 *)(base + L.yq);
    void *gws = base + L.gws;
    const size_t gws_bytes = w4a16_workspace_bytes(M, N, K, group);
    const __nv_bfloat16 *Wb = (const __nv_bfloat16 *)W, *Xb = (const __nv_bfloat16 *)X;

    cudaError_t e;
    if ((e = cudaMemsetAsync(losses, 0, sizeof(double) * n_alpha, stream)) != cudaSuccess) return e;
    if (gws_bytes && (e = cudaMemsetAsync(gws, 0, gws_bytes, stream)) != cudaSuccess) return e;
    act_kernel<<<(unsigned)((K + 255) / 256), 256, 0, stream>>>(Xb, (int)M, (int)K, act);
    ref_gemm_kernel<<<dim3((unsigned)((N + 63) / 64), (unsigned)((M + 63) / 64)), 256, 0, stream>>>(
        Xb, Wb, (int)M, (int)N, (int)K, yref);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const int64_t MK = M * K, MN = M * N;
    const unsigned ew_blocks = (unsigned)std::min<int64_t>((MK + 255) / 256, 148 * 16);
    const unsigned sq_blocks = (unsigned)std::min<int64_t>((MN + 255) / 256, 148 * 8);
    for (int i = 0; i < n_alpha; ++i) {
        scale_kernel<<<1, 1024, 0, stream>>>(act, (int)K, i, nullptr, n_alpha, s);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        if ((e = launch_quant_pack(W, N, K, group, mode, s, q, sc, z, stream)) != cudaSuccess) return e;
        xdiv_kernel<<<ew_blocks, 256, 0, stream>>>(Xb, s, MK, (int)K, xs);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
        const w4_status st = w4a16_gemm(xs, M, N, K, q, sc, z, group, mode, yq, gws, gws_bytes, (w4_stream_t)stream);
        if (st != W4_OK) return cudaErrorLaunchFailure;
        sqerr_kernel<<<sq_blocks, 256, 0, stream>>>(yref, yq, MN, losses + i);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    finish_kernel<<<1, 32, 0, stream>>>(losses, n_alpha, (double)MN, best);
    scale_kernel<<<1, 1024, 0, stream>>>(act, (int)K, 0, best, n_alpha, s_best);
    return cudaGetLastError();
}

}  // namespace w4
