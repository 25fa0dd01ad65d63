// w4a16_gemm_noalloc: the W4A16 product for callers that cannot allocate
// device memory.
//
// Who needs it: code that runs where cudaMalloc is not available or not
// allowed -- under a framework whose caching allocator owns all device memory
// and forbids side allocations, in a real-time or embedded host that freezes
// its memory map after start-up, or in a plug-in that receives only its input
// and output buffers.  w4a16_gemm needs a caller-provided workspace for its split-K
// shapes; this entry point uses a fixed scratch array that the library itself
// owns instead, so the caller passes only inputs and outputs.
//
// The scratch is a file-scope __device__ array of W4_NOALLOC_SCRATCH_BYTES.
// Every GPU that loads the library holds it until the process exits.  In host
// code its name is a host-side stand-in, not a device address: the address is
// obtained with cudaGetSymbolAddress once per device, with that device
// current, on the first call made on that device; make that first call
// before any stream capture on the device.  All calls share the one
// array and it keeps the last call's contents, so each call first clears the
// part that must start at zero (the split-K tile counters) with
// cudaMemsetAsync on the caller's stream.  Two calls whose work overlaps on
// the GPU (different streams without ordering, or different host threads)
// race on the array and give wrong results; calls on one stream are ordered
// and safe.
#include "common.cuh"

#include <atomic>

static __device__ __align__(256) unsigned char g_noalloc_scratch[W4_NOALLOC_SCRATCH_BYTES];

namespace {

std::atomic<void *> g_scratch_addr[w4::kMaxDevices];

// Device address of the scratch array on the current device, resolved on the
// first call for that device.
cudaError_t scratch_address(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= w4::kMaxDevices) return cudaErrorInvalidDevice;
    void *p = g_scratch_addr[dev].load(std::memory_order_acquire);
    if (!p) {
        e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
        if (e != cudaSuccess) return e;
        g_scratch_addr[dev].store(p, std::memory_order_release);
    }
    *out = p;
    return cudaSuccess;
}

bool aligned(const void *p, size_t a) { return ((uintptr_t)p % a) == 0; }

bool fits(int64_t a, int64_t b) { return a > 0 && b > 0 && a <= INT64_MAX / b; }

// The argument checks of w4a16_gemm, repeated here so that a call rejected for
// its arguments launches nothing (not even the counter clear).
bool args_ok(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight, const void *scales,
             const uint32_t *qzeros, int group, int mode, const void *Y)
{
    const bool f32 = (mode & W4_OUT_F32) != 0;
    mode &= ~(W4_WEIGHTS_STATIC | W4_OUT_F32 | W4_REPACKED);
    if (!X || !qweight || !scales || !Y) return false;
    if (!(group == 32 || group == 64 || group == 128) || !(mode == W4_SYM || mode == W4_ASYM)) return false;
    if (M < 1 || N < 1 || K < group || K % group != 0 || !fits(M, K) || !fits(N, K) || !fits(M, N)) return false;
    if ((mode == W4_ASYM) != (qzeros != nullptr)) return false;
    if (!aligned(X, 16) || !aligned(qweight, 16) || !aligned(scales, 2) || !aligned(Y, f32 ? 4 : 2)) return false;
    if (qzeros && !aligned(qzeros, 4)) return false;
    return true;
}

}  // namespace

extern "C" w4_status w4a16_gemm_noalloc(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                                        const void *scales, const uint32_t *qzeros, int group, int mode, void *Y,
                                        w4_stream_t stream)
{
    if (!args_ok(X, M, N, K, qweight, scales, qzeros, group, mode, Y)) return W4_ERR_INVALID_ARG;
    // every rejection happens before anything is enqueued, the counter clear included
    if (!w4::gemm_shape_supported(M, N, K)) return W4_ERR_UNSUPPORTED;
    const size_t need = w4a16_workspace_bytes(M, N, K, group);
    if (need > (size_t)W4_NOALLOC_SCRATCH_BYTES) return W4_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (need > 0) {
        if (scratch_address(&scratch) != cudaSuccess) return W4_ERR_CUDA;
        size_t off = 0, bytes = 0;
        w4::tc_workspace_counters(M, N, K, &off, &bytes);
        if (bytes > 0 &&
            cudaMemsetAsync((uint8_t *)scratch + off, 0, bytes, (cudaStream_t)stream) != cudaSuccess)
            return W4_ERR_CUDA;
    }
    return w4a16_gemm(X, M, N, K, qweight, scales, qzeros, group, mode, Y, scratch,
                      need > 0 ? (size_t)W4_NOALLOC_SCRATCH_BYTES : 0, stream);
}
