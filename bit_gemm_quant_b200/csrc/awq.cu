// w4_awq_search: the AWQ smoothing-scale search on the GPU.
//
// Method: page 2 (learn.longtimenohack.com/chasing/pages/quantization.html),
// AWQ section, the awq_search_scale listing: act = the mean magnitude of each
// input channel over the calibration rows; for alpha on an even grid over
// [0, 1], s = act^alpha / mean(act^alpha); quantize and dequantize W * s; the
// loss is mean((W X^T - (W^ / s) X^T)^2); keep the alpha with the smallest
// loss.  The exact readings are stated in include/w4.h.
//
// Every step runs in this library's kernels: once per search the channel
// magnitudes, the reference product W X^T (bf16 tensor-core MMAs, fp32
// accumulation), the scale vectors of all alphas (one CTA per alpha) and the
// activations divided by each of them; then per alpha w4_quant_pack with the
// fold, w4a16_gemm on the divided activations (the product (W^/s) X^T as the
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

// s_i[k] = fl32(act[k]^alpha_i / mean_k act^alpha_i), alpha_i = i / (n_alpha - 1):
// CTA i (1024 threads) writes the vector of alpha_i to s + i K.
__global__ void __launch_bounds__(1024) scale_kernel(const double *__restrict__ act, int K, int n_alpha,
                                                     float *__restrict__ s)
{
    __shared__ double red[32];
    const int i = blockIdx.x;
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
    for (int k = threadIdx.x; k < K; k += blockDim.x) s[(size_t)i * K + k] = (float)(pow(act[k], alpha) / mean);
}

// s_best = the vector of the best alpha
__global__ void pick_kernel(const float *__restrict__ s, int K, const int *__restrict__ best, float *__restrict__ s_best)
{
    const float *src = s + (size_t)(*best) * K;
    for (int k = blockIdx.x * blockDim.x + threadIdx.x; k < K; k += gridDim.x * blockDim.x) s_best[k] = src[k];
}

// Xs_i = bf16(fl32(x) / s_i[k]) (IEEE division) for every alpha i: Xs + i M K.
__global__ void xdiv_kernel(const __nv_bfloat16 *__restrict__ X, const float *__restrict__ s, int64_t MK, int K,
                            int n_alpha, __nv_bfloat16 *__restrict__ Xs)
{
    const int64_t total = MK * n_alpha;
    for (int64_t e = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; e < total; e += (int64_t)gridDim.x * blockDim.x) {
        const int64_t i = e / MK, j = e - i * MK;
        Xs[e] = __float2bfloat16_rn(__fdiv_rn(__bfloat162float(X[j]), s[i * K + j % K]));
    }
}

__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], const uint32_t (&b)[2])
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b[0]), "r"(b[1]));
}

// Y[m][n] = sum_k x[m][k] * w[n][k]: bf16 MMAs with fp32 accumulation.  A CTA
// (4 warps) computes 64 rows x 64 channels, a warp 32 x 32, over 32-wide
// k-slices staged in shared memory (rows padded to 80 bytes: the fragment
// reads of the 8 rows of a quad land on distinct banks).  K is a multiple of 32.
__global__ void __launch_bounds__(128) ref_gemm_kernel(const __nv_bfloat16 *__restrict__ X,
                                                       const __nv_bfloat16 *__restrict__ W, int M, int N, int K,
                                                       float *__restrict__ Y)
{
    __shared__ __align__(16) __nv_bfloat16 xs[64][40], ws[64][40];
    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5, g = lane >> 2, t = lane & 3;
    const int m0 = blockIdx.y * 64, n0 = blockIdx.x * 64;
    const int wm = (warp >> 1) * 32, wn = (warp & 1) * 32;
    float acc[2][4][4];
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j)
#pragma unroll
            for (int e = 0; e < 4; ++e) acc[i][j][e] = 0.f;
    for (int k0 = 0; k0 < K; k0 += 32) {
        for (int e = tid; e < 256; e += 128) {   // 64 rows x 32 k of X and of W, 16 bytes a thread
            const int r = e >> 2, c = (e & 3) * 8;
            const int m = m0 + r, n = n0 + r;
            uint4 xv = make_uint4(0u, 0u, 0u, 0u), wv = xv;
            if (m < M) xv = *(const uint4 *)(X + (size_t)m * K + k0 + c);
            if (n < N) wv = *(const uint4 *)(W + (size_t)n * K + k0 + c);
            *(uint4 *)&xs[r][c] = xv;
            *(uint4 *)&ws[r][c] = wv;
        }
        __syncthreads();
#pragma unroll
        for (int kk = 0; kk < 32; kk += 16) {
            uint32_t a[2][4], b[4][2];
#pragma unroll
            for (int i = 0; i < 2; ++i) {
                const int r = wm + 16 * i + g;
                a[i][0] = *(const uint32_t *)&xs[r][kk + 2 * t];
                a[i][1] = *(const uint32_t *)&xs[r + 8][kk + 2 * t];
                a[i][2] = *(const uint32_t *)&xs[r][kk + 2 * t + 8];
                a[i][3] = *(const uint32_t *)&xs[r + 8][kk + 2 * t + 8];
            }
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int c = wn + 8 * j + g;
                b[j][0] = *(const uint32_t *)&ws[c][kk + 2 * t];
                b[j][1] = *(const uint32_t *)&ws[c][kk + 2 * t + 8];
            }
#pragma unroll
            for (int i = 0; i < 2; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) mma_16816(acc[i][j], a[i], b[j]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 2; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int m = m0 + wm + 16 * i + g, n = n0 + wn + 8 * j + 2 * t;
            if (m < M && n < N) Y[(size_t)m * N + n] = acc[i][j][0];
            if (m < M && n + 1 < N) Y[(size_t)m * N + n + 1] = acc[i][j][1];
            if (m + 8 < M && n < N) Y[(size_t)(m + 8) * N + n] = acc[i][j][2];
            if (m + 8 < M && n + 1 < N) Y[(size_t)(m + 8) * N + n + 1] = acc[i][j][3];
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

AwqLayout awq_layout(int64_t M, int64_t N, int64_t K, int group, int mode, int n_alpha)
{
    AwqLayout L;
    const int64_t G = K / group;
    size_t o = 0;
    L.act = o; o += align256((size_t)K * 8);
    L.s = o; o += align256((size_t)n_alpha * K * 4);            // every alpha's scale vector
    L.xs = o; o += align256((size_t)n_alpha * M * K * 2);       // X divided by each of them
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

size_t awq_workspace_bytes(int64_t M, int64_t N, int64_t K, int group, int mode, int n_alpha)
{
    return awq_layout(M, N, K, group, mode, n_alpha).total;
}

cudaError_t launch_awq_search(const void *W, const void *X, int64_t N, int64_t K, int64_t M, int group, int mode,
                              int n_alpha, double *losses, int *best, float *s_best, void *ws, cudaStream_t stream)
{
    const AwqLayout L = awq_layout(M, N, K, group, mode, n_alpha);
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
    ref_gemm_kernel<<<dim3((unsigned)((N + 63) / 64), (unsigned)((M + 63) / 64)), 128, 0, stream>>>(
        Xb, Wb, (int)M, (int)N, (int)K, yref);
    scale_kernel<<<(unsigned)n_alpha, 1024, 0, stream>>>(act, (int)K, n_alpha, s);
    const int64_t MK = M * K, MN = M * N;
    xdiv_kernel<<<(unsigned)std::min<int64_t>((MK * n_alpha + 255) / 256, 148 * 16), 256, 0, stream>>>(
        Xb, s, MK, (int)K, n_alpha, xs);
    if ((e = cudaGetLastError()) != cudaSuccess) return e;
    const unsigned sq_blocks = (unsigned)std::min<int64_t>((MN + 255) / 256, 148 * 8);
    for (int i = 0; i < n_alpha; ++i) {
        if ((e = launch_quant_pack(W, N, K, group, mode, s + (size_t)i * K, q, sc, z, stream)) != cudaSuccess)
            return e;
        const w4_status st = w4a16_gemm(xs + (size_t)i * MK, M, N, K, q, sc, z, group, mode, yq, gws, gws_bytes,
                                        (w4_stream_t)stream);
        if (st != W4_OK) return cudaErrorLaunchFailure;
        sqerr_kernel<<<sq_blocks, 256, 0, stream>>>(yref, yq, MN, losses + i);
        if ((e = cudaGetLastError()) != cudaSuccess) return e;
    }
    finish_kernel<<<1, 32, 0, stream>>>(losses, n_alpha, (double)MN, best);
    pick_kernel<<<(unsigned)std::min<int64_t>((K + 255) / 256, 148), 256, 0, stream>>>(s, (int)K, best, s_best);
    return cudaGetLastError();
}

}  // namespace w4
