// extern "C" entry points of libw4 (declared in include/w4.h): argument
// validation on the host, then dispatch to the kernels.  Nothing here
// allocates device memory or synchronizes a stream.
#include "common.cuh"

namespace {

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool group_ok(int g) { return g == 32 || g == 64 || g == 128; }

bool mode_ok(int m) { return m == W4_SYM || m == W4_ASYM; }

// int64 products used for sizes must not overflow
bool fits(int64_t a, int64_t b) { return a > 0 && b > 0 && a <= INT64_MAX / b; }

}  // namespace

namespace w4 {

namespace {
std::atomic<uint64_t> g_wait_limit_ns{kDefaultWaitNs};
std::atomic<int> g_stall_first_wait{0};
}

uint64_t wait_limit_ns()
{
    return g_wait_limit_ns.load(std::memory_order_relaxed) |
           (g_stall_first_wait.load(std::memory_order_relaxed) ? kStallFirstWait : 0);
}

bool gemm_shape_supported(int64_t M, int64_t N, int64_t K)
{
    if (M <= kGemvMaxM) return N <= INT32_MAX - 16 && K <= INT32_MAX && M * K <= INT32_MAX;
    // tensor-core path: 32-bit indices, TMA extents
    return M <= INT32_MAX && N <= INT32_MAX && K <= INT32_MAX && M * K <= INT32_MAX &&
           (int64_t)N * K / 8 <= INT32_MAX * 4LL;
}

}  // namespace w4

extern "C" {

const char *w4_status_string(int status)
{
    switch (status) {
    case W4_OK: return "W4_OK";
    case W4_ERR_INVALID_ARG: return "W4_ERR_INVALID_ARG: null or misaligned pointer, bad size, group or mode";
    case W4_ERR_UNSUPPORTED: return "W4_ERR_UNSUPPORTED: well-formed request outside what the kernels cover";
    case W4_ERR_CUDA: return "W4_ERR_CUDA: a CUDA runtime call or kernel launch failed";
    default: return "unknown w4 status";
    }
}

int w4_layout_version(void) { return W4_LAYOUT_VERSION; }

w4_status w4_quant_pack(const void *W, int64_t N, int64_t K, int group, int mode, const float *s,
                        uint32_t *qweight, void *scales, uint32_t *qzeros, w4_stream_t stream)
{
    if (!W || !qweight || !scales) return W4_ERR_INVALID_ARG;
    if (!group_ok(group) || !mode_ok(mode)) return W4_ERR_INVALID_ARG;
    if (N < 1 || K < 8 || K % group != 0 || !fits(N, K)) return W4_ERR_INVALID_ARG;
    if (N > INT32_MAX - 65536 || K > INT32_MAX - 65536) return W4_ERR_UNSUPPORTED;   // 32-bit row / column indices
    if ((mode == W4_ASYM) != (qzeros != nullptr)) return W4_ERR_INVALID_ARG;
    if (!aligned(W, 32) || !aligned(qweight, 16) || !aligned(scales, 2)) return W4_ERR_INVALID_ARG;
    if (s && !aligned(s, 16)) return W4_ERR_INVALID_ARG;
    if (qzeros && !aligned(qzeros, 4)) return W4_ERR_INVALID_ARG;
    const cudaError_t e =
        w4::launch_quant_pack(W, N, K, group, mode, s, qweight, scales, qzeros, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_fp4_quant(const void *W, int64_t N, int64_t K, int kind, uint8_t *codes, uint8_t *scales,
                       w4_stream_t stream)
{
    if (!W || !codes || !scales) return W4_ERR_INVALID_ARG;
    if (kind != W4_NVFP4 && kind != W4_MXFP4) return W4_ERR_INVALID_ARG;
    const int64_t B = kind == W4_NVFP4 ? 16 : 32;
    if (N < 1 || K < B || K % B != 0 || !fits(N, K)) return W4_ERR_INVALID_ARG;
    if (!aligned(W, 16) || !aligned(codes, 16)) return W4_ERR_INVALID_ARG;
    const cudaError_t e = w4::launch_fp4_quant(W, N, K, kind, codes, scales, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

size_t w4_repacked_words(int64_t N, int64_t K)
{
    if (N < 1 || K < 256 || K % 256 != 0 || !fits(N + 15, K)) return 0;
    return (size_t)((N + 15) / 16 * 16) * (size_t)(K / 8);
}

w4_status w4_repack(const uint32_t *qweight, int64_t N, int64_t K, uint32_t *out, w4_stream_t stream)
{
    if (!qweight || !out) return W4_ERR_INVALID_ARG;
    if (N < 1 || K < 256 || !fits(N + 15, K)) return W4_ERR_INVALID_ARG;
    if (K % 256 != 0) return W4_ERR_UNSUPPORTED;
    if (!aligned(qweight, 16) || !aligned(out, 16)) return W4_ERR_INVALID_ARG;
    const cudaError_t e = w4::launch_repack(qweight, N, K, out, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

size_t w4_gptq_workspace_bytes(int64_t N, int64_t K, int group)
{
    if (N < 1 || K < 32 || !group_ok(group) || K % group != 0 || K > 16384 || !fits(N, K)) return 0;
    return w4::gptq_workspace_bytes(N, K, group);
}

w4_status w4_gptq(const void *W, const void *X, int64_t N, int64_t K, int64_t M, int group, int mode,
                  uint32_t *qweight, void *scales, uint32_t *qzeros, void *workspace, size_t workspace_bytes,
                  w4_stream_t stream)
{
    if (!W || !X || !qweight || !scales || !workspace) return W4_ERR_INVALID_ARG;
    if (!group_ok(group) || !mode_ok(mode)) return W4_ERR_INVALID_ARG;
    if (N < 1 || M < 1 || K < 32 || K % group != 0 || !fits(N, K) || !fits(M, K)) return W4_ERR_INVALID_ARG;
    if ((mode == W4_ASYM) != (qzeros != nullptr)) return W4_ERR_INVALID_ARG;
    if (!aligned(W, 2) || !aligned(X, 2) || !aligned(qweight, 4) || !aligned(scales, 2) || !aligned(workspace, 256))
        return W4_ERR_INVALID_ARG;
    if (qzeros && !aligned(qzeros, 4)) return W4_ERR_INVALID_ARG;
    if (K > 16384 || N > INT32_MAX || M > INT32_MAX) return W4_ERR_UNSUPPORTED;
    if (workspace_bytes < w4::gptq_workspace_bytes(N, K, group)) return W4_ERR_INVALID_ARG;
    const cudaError_t e = w4::launch_gptq(W, X, N, K, M, group, mode, qweight, scales, qzeros, workspace,
                                          (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_f32_to_bf16(const float *src, int64_t n, void *dst, w4_stream_t stream)
{
    if (!src || !dst || n < 1) return W4_ERR_INVALID_ARG;
    if (!aligned(src, 4) || !aligned(dst, 2)) return W4_ERR_INVALID_ARG;
    const cudaError_t e = w4::launch_f32_to_bf16(src, n, dst, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_mxfp8_quant(const void *X, int64_t M, int64_t K, uint8_t *codes, uint8_t *scales, int scale_layout,
                         w4_stream_t stream)
{
    if (!X || !codes || !scales) return W4_ERR_INVALID_ARG;
    if (scale_layout != W4_MX_SCALES_ROWS && scale_layout != W4_MX_SCALES_MMA) return W4_ERR_INVALID_ARG;
    if (M < 1 || K < 32 || K % 32 != 0 || !fits(M, K)) return W4_ERR_INVALID_ARG;
    if (scale_layout == W4_MX_SCALES_MMA && K % 128 != 0) return W4_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(codes, 16)) return W4_ERR_INVALID_ARG;
    if (scale_layout == W4_MX_SCALES_MMA && !aligned(scales, 16)) return W4_ERR_INVALID_ARG;
    if (!fits(w4::mx_padded_rows(M), K)) return W4_ERR_INVALID_ARG;
    const cudaError_t e = w4::launch_mxfp8_quant(X, M, K, codes, scales, scale_layout, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

w4_status w4_mx_scale_layout(const uint8_t *src, int64_t R, int64_t K, uint8_t *dst, w4_stream_t stream)
{
    if (!src || !dst) return W4_ERR_INVALID_ARG;
    if (R < 1 || K < 128 || K % 128 != 0 || !fits(R, K) || !fits(w4::mx_padded_rows(R), K)) return W4_ERR_INVALID_ARG;
    if (!aligned(src, 4) || !aligned(dst, 16)) return W4_ERR_INVALID_ARG;
    const cudaError_t e = w4::launch_mx_scale_layout(src, R, K, dst, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

namespace {
bool mx_shape_ok(int64_t M, int64_t N, int64_t K)
{
    return M >= 1 && N >= 1 && K >= 128 && K % 128 == 0 && fits(M, K) && fits(N, K) && fits(M, N);
}
// 32-bit indices in the kernel (rows, columns, split partial offsets use size_t)
bool mx_shape_supported(int64_t M, int64_t N, int64_t K)
{
    return M <= INT32_MAX - 256 && N <= INT32_MAX - 128 && K <= INT32_MAX && M * K <= (int64_t)1 << 40 &&
           N * K <= (int64_t)1 << 40;
}
}  // namespace

w4_status w4_mx_gemm(const uint8_t *x_codes, const uint8_t *x_scales, int64_t M, int64_t N, int64_t K,
                     const uint8_t *w_codes, const uint8_t *w_scales, void *Y, int flags, w4_stream_t stream)
{
    if (!x_codes || !x_scales || !w_codes || !w_scales || !Y) return W4_ERR_INVALID_ARG;
    if ((flags & ~W4_WEIGHTS_STATIC) != 0) return W4_ERR_INVALID_ARG;
    if (!mx_shape_ok(M, N, K)) return W4_ERR_INVALID_ARG;
    if (!aligned(x_codes, 16) || !aligned(x_scales, 16) || !aligned(w_codes, 32) || !aligned(w_scales, 16) ||
        !aligned(Y, 2))
        return W4_ERR_INVALID_ARG;
    if (!mx_shape_supported(M, N, K)) return W4_ERR_UNSUPPORTED;
    const cudaError_t e = w4::launch_mx_gemm(x_codes, x_scales, M, N, K, w_codes, w_scales, Y,
                                             (flags & W4_WEIGHTS_STATIC) != 0, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

size_t w4a16_workspace_bytes(int64_t M, int64_t N, int64_t K, int group)
{
    (void)group;
    if (M <= w4::kGemvMaxM || M < 1 || N < 1 || K < 1) return 0;
    return w4::tc_workspace_bytes(M, N, K);
}

w4_status w4a16_gemm(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                     const void *scales, const uint32_t *qzeros, int group, int mode, void *Y,
                     void *workspace, size_t workspace_bytes, w4_stream_t stream)
{
    const bool weights_static = (mode & W4_WEIGHTS_STATIC) != 0;
    const bool y_f32 = (mode & W4_OUT_F32) != 0;
    const bool repacked = (mode & W4_REPACKED) != 0;
    mode &= ~(W4_WEIGHTS_STATIC | W4_OUT_F32 | W4_REPACKED);
    if (!X || !qweight || !scales || !Y) return W4_ERR_INVALID_ARG;
    if (!group_ok(group) || !mode_ok(mode)) return W4_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < group || K % group != 0 || !fits(M, K) || !fits(N, K) || !fits(M, N))
        return W4_ERR_INVALID_ARG;
    if ((mode == W4_ASYM) != (qzeros != nullptr)) return W4_ERR_INVALID_ARG;
    if (!aligned(X, 16) || !aligned(qweight, 16) || !aligned(scales, 2) || !aligned(Y, y_f32 ? 4 : 2))
        return W4_ERR_INVALID_ARG;
    if (qzeros && !aligned(qzeros, 4)) return W4_ERR_INVALID_ARG;
    const size_t need = w4a16_workspace_bytes(M, N, K, group);
    if (need > workspace_bytes || (need > 0 && (!workspace || !aligned(workspace, 256))))
        return W4_ERR_INVALID_ARG;
    if (!w4::gemm_shape_supported(M, N, K)) return W4_ERR_UNSUPPORTED;
    if (repacked && (M > w4::kGemvMaxM || K % 256 != 0)) return W4_ERR_UNSUPPORTED;
    cudaError_t e;
    if (M <= w4::kGemvMaxM)
        e = w4::launch_gemv(X, M, N, K, qweight, scales, qzeros, group, mode, weights_static, y_f32, repacked, Y,
                            (cudaStream_t)stream);
    else
        e = w4::launch_gemm_tc(X, M, N, K, qweight, scales, qzeros, group, mode, y_f32, Y, workspace,
                               (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

size_t w4_awq_workspace_bytes(int64_t M, int64_t N, int64_t K, int group, int mode, int n_alpha)
{
    if (M < 1 || N < 1 || K < 1 || !group_ok(group) || !mode_ok(mode) || K % group != 0) return 0;
    if (n_alpha < 2 || n_alpha > 4096 || !fits(M, K) || !fits(M * K, n_alpha)) return 0;
    return w4::awq_workspace_bytes(M, N, K, group, mode, n_alpha);
}

w4_status w4_awq_search(const void *W, const void *X, int64_t N, int64_t K, int64_t M, int group, int mode,
                        int n_alpha, double *losses, int *best, float *s_best, void *workspace,
                        size_t workspace_bytes, w4_stream_t stream)
{
    if (!W || !X || !losses || !best || !s_best || !workspace) return W4_ERR_INVALID_ARG;
    if (!group_ok(group) || !mode_ok(mode) || n_alpha < 2 || n_alpha > 4096) return W4_ERR_INVALID_ARG;
    if (M < 1 || N < 1 || K < group || K % group != 0 || !fits(M, K) || !fits(N, K) || !fits(M, N))
        return W4_ERR_INVALID_ARG;
    if (!aligned(W, 32) || !aligned(X, 16) || !aligned(losses, 8) || !aligned(best, 4) || !aligned(s_best, 16) ||
        !aligned(workspace, 256))
        return W4_ERR_INVALID_ARG;
    if (!fits(M * K, n_alpha) || workspace_bytes < w4::awq_workspace_bytes(M, N, K, group, mode, n_alpha))
        return W4_ERR_INVALID_ARG;
    if (M > INT32_MAX || N > INT32_MAX - 16 || K > INT32_MAX || M * K > INT32_MAX || M * N > INT32_MAX)
        return W4_ERR_UNSUPPORTED;
    const cudaError_t e = w4::launch_awq_search(W, X, N, K, M, group, mode, n_alpha, losses, best, s_best,
                                                workspace, (cudaStream_t)stream);
    return e == cudaSuccess ? W4_OK : W4_ERR_CUDA;
}

void w4_set_wait_limit_ns(uint64_t ns)
{
    ns = ns == 0 ? w4::kDefaultWaitNs : ns;
    w4::g_wait_limit_ns.store(ns > w4::kDefaultWaitNs ? w4::kDefaultWaitNs : ns, std::memory_order_relaxed);
}

void w4_test_stall_first_wait(int on) { w4::g_stall_first_wait.store(on ? 1 : 0, std::memory_order_relaxed); }

w4_status w4_device_error(int *code)
{
    if (!code) return W4_ERR_INVALID_ARG;
    if (cudaDeviceSynchronize() != cudaSuccess) return W4_ERR_CUDA;
    const int v = w4::read_and_clear_device_error();
    if (v < 0) return W4_ERR_CUDA;
    *code = v;
    return W4_OK;
}

}  // extern "C"
