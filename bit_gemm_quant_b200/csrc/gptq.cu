// w4_gptq: GPTQ -- Hessian-aware INT4 rounding with error feedback -- into
// the library's packed format.
//
// Method: page 5 (ai-infra.cypggs.com .../02-core-ideas) section 2.5: columns
// are quantized one at a time and each column's rounding error, scaled by the
// upper Cholesky factor U of the inverse Hessian (H^-1 = U^T U), is fed back
// into every later column: e = (w_j - w^_j) / U[j][j], w_k -= e U[j][k] for
// k > j.  Page 3 (blog.freezetheflame.cc quantization deep dive) section 3.1:
// H = 2 X^T X over the calibration rows, damped by lambda = 0.01 trace / K; a
// group's scale comes from its columns when its first column is reached.  The
// grid of each group follows page 5 section 2.2 exactly as w4_quant_pack does.
// The exact semantics are spelled out in include/w4.h.
//
// B200 design, all arithmetic in fp64 (the factorization of a damped Hessian
// loses about log10(cond) digits, and fp64 keeps the result within rounding of
// the fp64 definition):
//   1. lambda: one CTA sums x^2 over the calibration rows (fixed order);
//   2. H: a symmetric rank-M product, written in REVERSED index order
//      (Hr[a][b] = H[K-1-a][K-1-b]), lower triangle only;
//   3. Hr = L L^T by a blocked right-looking Cholesky (32-wide blocks: one
//      CTA factors the diagonal block, a panel kernel solves the column below
//      it, a tiled kernel updates the trailing lower triangle);
//   4. L^-1 by blocked forward substitution: the diagonal blocks first, then
//      one launch per block diagonal.  With J the index reversal,
//      J H J = L L^T gives H = (J L J)(J L J)^T with J L J upper triangular,
//      so H^-1 = (J L^-1 J)^T (J L^-1 J): U = J L^-1 J, i.e.
//      U[j][k] = Linv[K-1-j][K-1-k] -- one Cholesky and one triangular
//      inverse instead of an explicit inverse and a second Cholesky;
//   5. the column loop: at each group's first column one launch sets every
//      row's grid from the group's current values; then one launch per block
//      of 32 columns: a CTA owns 64 rows (rows are independent given U); 64
//      of its threads run the block's 32 sequential steps for one row each in
//      registers (the code, the error, the updates of the block's later
//      columns), and then all 256 threads apply the block's 32 errors to this
//      CTA's slice of the later columns (the "lazy batch" form of the same
//      updates: only the summation order differs);
//   6. the zero-points are packed 8 per word at the end.
// With no calibration signal (trace 0) H is singular; as in the definition, U
// is then the identity: nothing is fed back and GPTQ is plain rounding.
#include "common.cuh"

namespace w4 {
namespace {

constexpr int kB = 32;               // block width (factorization and column loop)
constexpr int kRows = 64;            // rows of W per column-loop CTA
constexpr int kCols = 256;           // later columns per column-loop CTA

// ---------------------------------------------------------------- 1, 2 --

// lambda = 0.01 * trace(X^T X) / K = 0.01 * sum x^2 / K, one CTA, fixed order.
__global__ void __launch_bounds__(256) gptq_lambda_kernel(const __nv_bfloat16 *__restrict__ X, int64_t MK, int K,
                                                          double *__restrict__ lam)
{
    pdl_wait();
    pdl_launch_dependents();
    __shared__ double part[256];
    double s = 0.0;
    for (int64_t i = threadIdx.x; i < MK; i += 256) {
        const double x = (double)__bfloat162float(X[i]);
        s = fma(x, x, s);
    }
    part[threadIdx.x] = s;
    __syncthreads();
    for (int w = 128; w > 0; w >>= 1) {
        if (threadIdx.x < w) part[threadIdx.x] += part[threadIdx.x + w];
        __syncthreads();
    }
    if (threadIdx.x == 0) *lam = 0.01 * part[0] / (double)K;
}

// Hr[a][b] = 2 sum_m x[m][K-1-a] x[m][K-1-b] (+ lambda on the diagonal) for the
// 64 x 64 tile (blockIdx.y, blockIdx.x) of the lower triangle; each thread owns
// 4 x 4 outputs.
__global__ void __launch_bounds__(256) gptq_hessian_kernel(const __nv_bfloat16 *__restrict__ X, int M, int K,
                                                           const double *__restrict__ lam, double *__restrict__ Hr)
{
    pdl_wait();
    pdl_launch_dependents();
    const int ta = blockIdx.y, tb = blockIdx.x;
    if (tb > ta) return;                             // upper triangle: not needed
    __shared__ double xa[16][64], xb[16][64];
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double acc[4][4] = {};
    for (int m0 = 0; m0 < M; m0 += 16) {
        for (int e = threadIdx.x; e < 16 * 64; e += 256) {
            const int mm = e >> 6, c = e & 63;
            const int m = m0 + mm;
            const int ia = ta * 64 + c, ib = tb * 64 + c;
            xa[mm][c] = (m < M && ia < K) ? (double)__bfloat162float(X[(size_t)m * K + (K - 1 - ia)]) : 0.0;
            xb[mm][c] = (m < M && ib < K) ? (double)__bfloat162float(X[(size_t)m * K + (K - 1 - ib)]) : 0.0;
        }
        __syncthreads();
#pragma unroll 4
        for (int mm = 0; mm < 16; ++mm) {
            double va[4], vb[4];
#pragma unroll
            for (int i = 0; i < 4; ++i) va[i] = xa[mm][ty + 16 * i];
#pragma unroll
            for (int j = 0; j < 4; ++j) vb[j] = xb[mm][tx + 16 * j];
#pragma unroll
            for (int i = 0; i < 4; ++i)
#pragma unroll
                for (int j = 0; j < 4; ++j) acc[i][j] = fma(va[i], vb[j], acc[i][j]);
        }
        __syncthreads();
    }
    const double l = *lam;
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int a = ta * 64 + ty + 16 * i, b = tb * 64 + tx + 16 * j;
            if (a < K && b <= a) Hr[(size_t)a * K + b] = 2.0 * acc[i][j] + (a == b ? l : 0.0);
        }
}

// ------------------------------------------------------------------- 3 --

// Unblocked Cholesky of the diagonal block p (kB x kB, lower) in shared memory.
__global__ void __launch_bounds__(256) chol_diag_kernel(double *__restrict__ A, int K, int p, int *__restrict__ bad)
{
    pdl_wait();
    pdl_launch_dependents();
    __shared__ double a[kB][kB + 1];
    const int o = p * kB;
    for (int e = threadIdx.x; e < kB * kB; e += 256) {
        const int r = e / kB, c = e % kB;
        a[r][c] = c <= r ? A[(size_t)(o + r) * K + o + c] : 0.0;
    }
    __syncthreads();
    for (int c = 0; c < kB; ++c) {
        if (threadIdx.x == 0) {
            const double d = a[c][c];
            if (!(d > 0.0)) atomicExch(bad, 1);      // not positive definite (no calibration signal)
            a[c][c] = d > 0.0 ? sqrt(d) : 1.0;
        }
        __syncthreads();
        if (threadIdx.x > c && threadIdx.x < kB) a[threadIdx.x][c] /= a[c][c];
        __syncthreads();
        for (int e = threadIdx.x; e < kB * kB; e += 256) {
            const int r = e / kB, s = e % kB;
            if (s > c && s <= r) a[r][s] -= a[r][c] * a[s][c];
        }
        __syncthreads();
    }
    for (int e = threadIdx.x; e < kB * kB; e += 256) {
        const int r = e / kB, c = e % kB;
        if (c <= r) A[(size_t)(o + r) * K + o + c] = a[r][c];
    }
}

// The column of blocks below block p: row i solves x L_pp^T = a (forward
// substitution over the block's kB columns).
__global__ void __launch_bounds__(128) chol_panel_kernel(double *__restrict__ A, int K, int p)
{
    pdl_wait();
    pdl_launch_dependents();
    __shared__ double l[kB][kB + 1];
    const int o = p * kB;
    for (int e = threadIdx.x; e < kB * kB; e += 128) {
        const int r = e / kB, c = e % kB;
        l[r][c] = c <= r ? A[(size_t)(o + r) * K + o + c] : 0.0;
    }
    __syncthreads();
    const int i = o + kB + blockIdx.x * 128 + threadIdx.x;
    if (i >= K) return;
    double x[kB];
#pragma unroll
    for (int c = 0; c < kB; ++c) x[c] = A[(size_t)i * K + o + c];
#pragma unroll
    for (int c = 0; c < kB; ++c) {
        double v = x[c];
#pragma unroll
        for (int s = 0; s < c; ++s) v -= x[s] * l[c][s];
        x[c] = v / l[c][c];
    }
#pragma unroll
    for (int c = 0; c < kB; ++c) A[(size_t)i * K + o + c] = x[c];
}

// Trailing update of the lower triangle below and right of block p:
// A[i][j] -= sum_c L[i][o+c] L[j][o+c] on the 64 x 64 tile (blockIdx.y, blockIdx.x)
// of the trailing matrix.
__global__ void __launch_bounds__(256) chol_update_kernel(double *__restrict__ A, int K, int p)
{
    pdl_wait();
    pdl_launch_dependents();
    const int ti = blockIdx.y, tj = blockIdx.x;
    if (tj > ti) return;
    const int o = p * kB, t0 = o + kB;
    __shared__ double li[kB][64], lj[kB][64];
    for (int e = threadIdx.x; e < kB * 64; e += 256) {
        const int c = e / 64, r = e % 64;
        const int i = t0 + ti * 64 + r, j = t0 + tj * 64 + r;
        li[c][r] = i < K ? A[(size_t)i * K + o + c] : 0.0;
        lj[c][r] = j < K ? A[(size_t)j * K + o + c] : 0.0;
    }
    __syncthreads();
    const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
    double acc[4][4] = {};
#pragma unroll 4
    for (int c = 0; c < kB; ++c) {
        double va[4], vb[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) va[u] = li[c][ty + 16 * u];
#pragma unroll
        for (int v = 0; v < 4; ++v) vb[v] = lj[c][tx + 16 * v];
#pragma unroll
        for (int u = 0; u < 4; ++u)
#pragma unroll
            for (int v = 0; v < 4; ++v) acc[u][v] = fma(va[u], vb[v], acc[u][v]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
#pragma unroll
        for (int v = 0; v < 4; ++v) {
            const int i = t0 + ti * 64 + ty + 16 * u, j = t0 + tj * 64 + tx + 16 * v;
            if (i < K && j <= i) A[(size_t)i * K + j] -= acc[u][v];
        }
}

// ------------------------------------------------------------------- 4 --

// Inverse of every diagonal block (blockIdx.x = p): thread c solves L_pp x = e_c.
__global__ void __launch_bounds__(kB) trinv_diag_kernel(const double *__restrict__ L, int K,
                                                        double *__restrict__ Li)
{
    pdl_wait();
    pdl_launch_dependents();
    __shared__ double l[kB][kB + 1];
    const int o = blockIdx.x * kB;
    for (int r = 0; r < kB; ++r) l[r][threadIdx.x] = threadIdx.x <= r ? L[(size_t)(o + r) * K + o + threadIdx.x] : 0.0;
    __syncthreads();
    const int c = threadIdx.x;
    double x[kB];
#pragma unroll
    for (int r = 0; r < kB; ++r) {
        double v = (r == c) ? 1.0 : 0.0;
#pragma unroll
        for (int s = 0; s < r; ++s) v -= l[r][s] * x[s];
        x[r] = v / l[r][r];
    }
#pragma unroll
    for (int r = 0; r < kB; ++r) Li[(size_t)(o + r) * K + o + c] = r >= c ? x[r] : 0.0;
}

// Block diagonal d of the inverse: for p = blockIdx.x, q = p + d,
// Li[q][p] = -Li[q][q] * sum_{k=p}^{q-1} L[q][k] Li[k][p]  (kB x kB blocks).
__global__ void __launch_bounds__(256) trinv_offdiag_kernel(const double *__restrict__ L, int K, int d,
                                                            double *__restrict__ Li)
{
    pdl_wait();
    pdl_launch_dependents();
    const int p = blockIdx.x, q = p + d;
    __shared__ double a[kB][kB + 1], b[kB][kB + 1], t[kB][kB + 1];
    const int tr = threadIdx.x / 8, tc0 = (threadIdx.x % 8) * 4;     // 4 outputs per thread
    double acc[4] = {0.0, 0.0, 0.0, 0.0};
    for (int k = p; k < q; ++k) {
        for (int e = threadIdx.x; e < kB * kB; e += 256) {
            const int r = e / kB, c = e % kB;
            a[r][c] = L[(size_t)(q * kB + r) * K + k * kB + c];
            b[r][c] = Li[(size_t)(k * kB + r) * K + p * kB + c];
        }
        __syncthreads();
#pragma unroll 8
        for (int s = 0; s < kB; ++s) {
            const double av = a[tr][s];
#pragma unroll
            for (int u = 0; u < 4; ++u) acc[u] = fma(av, b[s][tc0 + u], acc[u]);
        }
        __syncthreads();
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) t[tr][tc0 + u] = acc[u];
    for (int e = threadIdx.x; e < kB * kB; e += 256) {
        const int r = e / kB, c = e % kB;
        a[r][c] = c <= r ? Li[(size_t)(q * kB + r) * K + q * kB + c] : 0.0;
    }
    __syncthreads();
    double out[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll 8
    for (int s = 0; s < kB; ++s) {
        const double av = a[tr][s];
#pragma unroll
        for (int u = 0; u < 4; ++u) out[u] = fma(av, t[s][tc0 + u], out[u]);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) Li[(size_t)(q * kB + tr) * K + p * kB + tc0 + u] = -out[u];
}

// ------------------------------------------------------------------- 5 --

__global__ void __launch_bounds__(256) gptq_load_kernel(const __nv_bfloat16 *__restrict__ W, int64_t n,
                                                        double *__restrict__ Wf)
{
    pdl_wait();
    pdl_launch_dependents();
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (int64_t)gridDim.x * blockDim.x)
        Wf[i] = (double)__bfloat162float(W[i]);
}

// The group grid from the group's current values (fp32 statistics, fp16
// scale saturated to 65504, zero-point from the fp16 scale), the rules of
// w4_quant_pack.
template <int MODE>
__device__ __forceinline__ void group_grid(float a, float mn, float mx, unsigned short &s16, int &zp)
{
    const float s32 = (MODE == W4_SYM) ? __fdiv_rn(a, 7.0f) : __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
    s16 = (s32 > 65504.0f) ? (unsigned short)0x7BFF : __half_as_ushort(__float2half_rn(s32));
    const float d = __half2float(__ushort_as_half(s16));
    if (MODE == W4_SYM) zp = 8;
    else zp = (d > 0.f) ? (int)fminf(fmaxf(rintf(__fdiv_rn(-mn, d)), 0.f), 15.f) : 0;
}

template <int MODE>
__device__ __forceinline__ int grid_code(float w32, float d, int zp)
{
    if (!(d > 0.f)) return MODE == W4_SYM ? 8 : 0;
    const float c = rintf(__fdiv_rn(w32, d));
    return MODE == W4_SYM ? (int)fminf(fmaxf(c, -8.f), 7.f) + 8 : (int)fminf(fmaxf(c + (float)zp, 0.f), 15.f);
}

// The grids of the group that starts at column j0, one thread per row, from
// the group's current values (every earlier column's feedback applied, none
// of the group's own).
template <int MODE>
__global__ void __launch_bounds__(256) gptq_grid_kernel(const double *__restrict__ Wf, int N, int K, int j0, int g,
                                                        unsigned short *__restrict__ scales,
                                                        uint8_t *__restrict__ zps)
{
    pdl_wait();
    pdl_launch_dependents();
    const int n = blockIdx.x * 256 + threadIdx.x;
    if (n >= N) return;
    const double *row = Wf + (size_t)n * K + j0;
    float a = 0.f, mn = 0.f, mx = 0.f;
    for (int k = 0; k < g; ++k) {
        const float x = __double2float_rn(row[k]);
        a = fmaxf(a, fabsf(x));
        mn = fminf(mn, x);
        mx = fmaxf(mx, x);
    }
    unsigned short s16;
    int zp;
    group_grid<MODE>(a, mn, mx, s16, zp);
    const int G = K / g;
    scales[(size_t)n * G + j0 / g] = s16;
    zps[(size_t)n * G + j0 / g] = (uint8_t)zp;
}

// Column block b (columns b*kB .. b*kB+kB-1) for rows [blockIdx.x*kRows, +kRows)
// and later columns [c0, c0 + kCols), c0 = (b+1)*kB + blockIdx.y*kCols.  The
// block lies inside one group (g is a multiple of kB), whose grid the grid
// kernel stored before.
template <int MODE>
__global__ void __launch_bounds__(256) gptq_block_kernel(double *__restrict__ Wf, const double *__restrict__ Li,
                                                         int N, int K, int b, int g, const int *__restrict__ bad,
                                                         uint32_t *__restrict__ qweight,
                                                         const unsigned short *__restrict__ scales,
                                                         const uint8_t *__restrict__ zps)
{
    pdl_wait();
    pdl_launch_dependents();
    __shared__ double u[kB][kB + 1];                 // U on the block: u[j][k] = U[j0+j][j0+k], k >= j
    __shared__ double e_s[kB][kRows + 1];            // errors of the block, [column][row]
    const int j0 = b * kB;
    const int G = K / g;
    const bool ident = *bad != 0;                    // no calibration signal: U = I
    for (int e = threadIdx.x; e < kB * kB; e += 256) {
        const int j = e / kB, k = e % kB;
        double v = 0.0;
        if (ident) v = (j == k) ? 1.0 : 0.0;
        else if (k >= j) v = Li[(size_t)(K - 1 - (j0 + j)) * K + (K - 1 - (j0 + k))];
        u[j][k] = v;
    }
    __syncthreads();
    const int r = threadIdx.x;
    const int n = blockIdx.x * kRows + r;
    if (r < kRows) {
        double er[kB];
        if (n < N) {
            double w[kB];
            const double *row = Wf + (size_t)n * K;
#pragma unroll
            for (int j = 0; j < kB; ++j) w[j] = row[j0 + j];
            const int gi = j0 / g;
            const unsigned short s16 = scales[(size_t)n * G + gi];
            const int zp = zps[(size_t)n * G + gi];
            const float d = __half2float(__ushort_as_half(s16));
            uint32_t words[kB / 8] = {};
#pragma unroll
            for (int j = 0; j < kB; ++j) {
                const int c = grid_code<MODE>(__double2float_rn(w[j]), d, zp);
                const double what = (double)(c - zp) * (double)d;
                const double ej = (w[j] - what) / u[j][j];
                er[j] = ej;
#pragma unroll
                for (int k = j + 1; k < kB; ++k) w[k] = fma(-ej, u[j][k], w[k]);
                const int e8 = j & 7;
                words[j >> 3] |= (uint32_t)c << (4 * (e8 >> 1) + ((e8 & 1) ? 16 : 0));
            }
            if (blockIdx.y == 0) {
#pragma unroll
                for (int t = 0; t < kB / 8; ++t) qweight[(size_t)n * (K / 8) + j0 / 8 + t] = words[t];
            }
        } else {
#pragma unroll
            for (int j = 0; j < kB; ++j) er[j] = 0.0;
        }
#pragma unroll
        for (int j = 0; j < kB; ++j) e_s[j][r] = er[j];
    }
    __syncthreads();
    // the block's errors applied to this CTA's slice of the later columns
    const int col = (b + 1) * kB + blockIdx.y * kCols + threadIdx.x;
    if (col >= K) return;
    double uc[kB];
#pragma unroll
    for (int j = 0; j < kB; ++j)
        uc[j] = ident ? 0.0 : Li[(size_t)(K - 1 - (j0 + j)) * K + (K - 1 - col)];
    const int rows = min(kRows, N - (int)blockIdx.x * kRows);
    for (int rr = 0; rr < rows; ++rr) {
        double acc = 0.0;
#pragma unroll
        for (int j = 0; j < kB; ++j) acc = fma(e_s[j][rr], uc[j], acc);
        double *p = Wf + (size_t)(blockIdx.x * kRows + rr) * K + col;
        *p -= acc;
    }
}

// ------------------------------------------------------------------- 6 --

__global__ void __launch_bounds__(256) gptq_pack_zeros_kernel(const uint8_t *__restrict__ zps, int N, int G,
                                                              uint32_t *__restrict__ qzeros)
{
    pdl_wait();
    pdl_launch_dependents();
    const int ZW = (G + 7) / 8;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < (int64_t)N * ZW;
         i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t n = i / ZW;
        const int w = (int)(i - n * ZW);
        uint32_t v = 0;
        for (int t = 0; t < 8 && w * 8 + t < G; ++t) v |= (uint32_t)(zps[n * G + w * 8 + t] & 15) << (4 * t);
        qzeros[i] = v;
    }
}

struct GptqWs {
    size_t lam, bad, hr, li, wf, zps, total;
};

GptqWs gptq_layout(int64_t N, int64_t K, int group)
{
    auto al = [](size_t x) { return (x + 255) & ~(size_t)255; };
    GptqWs w;
    w.lam = 0;
    w.bad = 256;
    w.hr = 512;
    w.li = w.hr + al((size_t)K * K * 8);
    w.wf = w.li + al((size_t)K * K * 8);
    w.zps = w.wf + al((size_t)N * K * 8);
    w.total = w.zps + al((size_t)N * (K / group));
    return w;
}

}  // namespace

size_t gptq_workspace_bytes(int64_t N, int64_t K, int group) { return gptq_layout(N, K, group).total; }

cudaError_t launch_gptq(const void *W, const void *X, int64_t N, int64_t K, int64_t M, int group, int mode,
                        uint32_t *qweight, void *scales, uint32_t *qzeros, void *ws, cudaStream_t stream)
{
    const GptqWs L = gptq_layout(N, K, group);
    uint8_t *base = (uint8_t *)ws;
    double *lam = (double *)(base + L.lam);
    int *bad = (int *)(base + L.bad);
    double *Hr = (double *)(base + L.hr);
    double *Li = (double *)(base + L.li);
    double *Wf = (double *)(base + L.wf);
    uint8_t *zps = base + L.zps;
    const int Ki = (int)K, Ni = (int)N, NB = Ki / kB;
    cudaError_t e;
    if ((e = cudaMemsetAsync(bad, 0, sizeof(int), stream)) != cudaSuccess) return e;
    // (the strictly upper triangle of Hr is never read: the factorization and
    // the inverse touch the lower triangle only)
    if ((e = cudaMemsetAsync(Li, 0, (size_t)K * K * 8, stream)) != cudaSuccess) return e;
    if ((e = launch_pdl(gptq_lambda_kernel, dim3(1), dim3(256), 0, stream, (const __nv_bfloat16 *)X, (int64_t)M * K,
                        Ki, lam)) != cudaSuccess)
        return e;
    const int T = (Ki + 63) / 64;
    if ((e = launch_pdl(gptq_hessian_kernel, dim3(T, T), dim3(256), 0, stream, (const __nv_bfloat16 *)X, (int)M, Ki,
                        (const double *)lam, Hr)) != cudaSuccess)
        return e;
    for (int p = 0; p < NB; ++p) {
        if ((e = launch_pdl(chol_diag_kernel, dim3(1), dim3(256), 0, stream, Hr, Ki, p, bad)) != cudaSuccess) return e;
        const int below = Ki - (p + 1) * kB;
        if (below <= 0) break;
        if ((e = launch_pdl(chol_panel_kernel, dim3((below + 127) / 128), dim3(128), 0, stream, Hr, Ki, p)) !=
            cudaSuccess)
            return e;
        const int tt = (below + 63) / 64;
        if ((e = launch_pdl(chol_update_kernel, dim3(tt, tt), dim3(256), 0, stream, Hr, Ki, p)) != cudaSuccess)
            return e;
    }
    if ((e = launch_pdl(trinv_diag_kernel, dim3(NB), dim3(kB), 0, stream, (const double *)Hr, Ki, Li)) != cudaSuccess)
        return e;
    for (int d = 1; d < NB; ++d)
        if ((e = launch_pdl(trinv_offdiag_kernel, dim3(NB - d), dim3(256), 0, stream, (const double *)Hr, Ki, d, Li)) !=
            cudaSuccess)
            return e;
    if ((e = launch_pdl(gptq_load_kernel, dim3(kNumSMs * 8), dim3(256), 0, stream, (const __nv_bfloat16 *)W,
                        (int64_t)N * K, Wf)) != cudaSuccess)
        return e;
    const unsigned rb = (unsigned)((N + kRows - 1) / kRows);
    for (int b = 0; b < NB; ++b) {
        if ((b * kB) % group == 0) {
            if (mode == W4_SYM)
                e = launch_pdl(gptq_grid_kernel<W4_SYM>, dim3((Ni + 255) / 256), dim3(256), 0, stream,
                               (const double *)Wf, Ni, Ki, b * kB, group, (unsigned short *)scales, zps);
            else
                e = launch_pdl(gptq_grid_kernel<W4_ASYM>, dim3((Ni + 255) / 256), dim3(256), 0, stream,
                               (const double *)Wf, Ni, Ki, b * kB, group, (unsigned short *)scales, zps);
            if (e != cudaSuccess) return e;
        }
        const int later = Ki - (b + 1) * kB;
        const unsigned cb = (unsigned)(later > 0 ? (later + kCols - 1) / kCols : 1);
        if (mode == W4_SYM)
            e = launch_pdl(gptq_block_kernel<W4_SYM>, dim3(rb, cb), dim3(256), 0, stream, Wf, (const double *)Li, Ni,
                           Ki, b, group, (const int *)bad, qweight, (const unsigned short *)scales,
                           (const uint8_t *)zps);
        else
            e = launch_pdl(gptq_block_kernel<W4_ASYM>, dim3(rb, cb), dim3(256), 0, stream, Wf, (const double *)Li,
                           Ni, Ki, b, group, (const int *)bad, qweight, (const unsigned short *)scales,
                           (const uint8_t *)zps);
        if (e != cudaSuccess) return e;
    }
    if (mode == W4_ASYM)
        return launch_pdl(gptq_pack_zeros_kernel, dim3(kNumSMs * 4), dim3(256), 0, stream, (const uint8_t *)zps, Ni,
                          Ki / group, qzeros);
    return cudaSuccess;
}

}  // namespace w4
