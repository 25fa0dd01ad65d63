// Shared helpers of libw4 (CUDA side only).
#pragma once

#include <cuda_runtime.h>
#include <cuda_fp16.h>
#include <cuda_bf16.h>
#include <stdint.h>

#include <atomic>
#include <utility>

#include "w4.h"

namespace w4 {

constexpr int kNumSMs = 148;             // B200

// Start fetching [p, p + bytes) from HBM into L2 (cp.async.bulk.prefetch); a
// hint only.  The range is shrunk to its 16-byte-aligned interior so it never
// leaves the array.
__device__ __forceinline__ void prefetch_l2(const void *p, size_t bytes)
{
    uintptr_t a = ((uintptr_t)p + 15) & ~(uintptr_t)15;
    const uintptr_t e = ((uintptr_t)p + bytes) & ~(uintptr_t)15;
    while (a < e) {
        const uint32_t n = (e - a) > (1u << 20) ? (1u << 20) : (uint32_t)(e - a);
        asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(a), "r"(n) : "memory");
        a += n;
    }
}

// Programmatic dependent launch.  Every kernel of the library is launched with
// programmatic stream serialization, so it may start while the previous kernel
// of the stream drains; it runs only set-up that touches no global memory (its
// shared-memory barriers, tensor-memory allocation, descriptor prefetch) before
// pdl_wait(), which returns once the previous kernel has completed and its
// writes are visible.  pdl_launch_dependents() then lets the next kernel start
// its own set-up.  A previous kernel that does not trigger releases the next
// one when it exits, so ordering against any other work on the stream is the
// same as without the attribute.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                       Args &&...args)
{
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// One output element of the product: bf16 (round to nearest even) or, with
// W4_OUT_F32, the fp32 sum itself.
__device__ __forceinline__ void store_y(void *Y, size_t idx, float v, int y_f32)
{
    if (y_f32) ((float *)Y)[idx] = v;
    else ((__nv_bfloat16 *)Y)[idx] = __float2bfloat16_rn(v);
}

__device__ __forceinline__ float bf16lo_to_f32(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16hi_to_f32(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }

// Launchers (host side), implemented in the kernel files.
cudaError_t launch_quant_pack(const void *W, int64_t N, int64_t K, int group, int mode, const float *s,
                              uint32_t *qweight, void *scales, uint32_t *qzeros, cudaStream_t stream);
cudaError_t launch_gemv(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                        const void *scales, const uint32_t *qzeros, int group, int mode, bool weights_static,
                        bool y_f32, bool repacked, void *Y, cudaStream_t stream);
// the GEMV's code layout: w4_repack (16-row x 256-k boxes stored contiguously)
cudaError_t launch_repack(const uint32_t *qweight, int64_t N, int64_t K, uint32_t *out, cudaStream_t stream);
// Batches up to this size run the GEMV (two MMA token groups of 8); larger ones
// the tensor-core kernel.
constexpr int64_t kGemvMaxM = 16;
// Shapes the product's kernels cannot index (32-bit indices, TMA extents).
bool gemm_shape_supported(int64_t M, int64_t N, int64_t K);
// Opt a kernel into `bytes` of dynamic shared memory on the current device.
// The attribute is per device, so the flag that skips repeated calls is kept
// per device too (an array indexed by the device ordinal).
constexpr int kMaxDevices = 64;
template <typename Kern>
cudaError_t set_smem_attr(Kern kern, int bytes, std::atomic<bool> (&done)[kMaxDevices])
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess) return e;
    if (dev < 0 || dev >= kMaxDevices) return cudaErrorInvalidDevice;
    if (done[dev].load(std::memory_order_acquire)) return cudaSuccess;
    e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
    if (e == cudaSuccess) done[dev].store(true, std::memory_order_release);
    return e;
}
cudaError_t launch_fp4_quant(const void *W, int64_t N, int64_t K, int kind, uint8_t *codes, uint8_t *scales,
                             cudaStream_t stream);
// GPTQ: workspace bytes and the whole procedure on `stream`
size_t gptq_workspace_bytes(int64_t N, int64_t K, int group);
cudaError_t launch_gptq(const void *W, const void *X, int64_t N, int64_t K, int64_t M, int group, int mode,
                        uint32_t *qweight, void *scales, uint32_t *qzeros, void *ws, cudaStream_t stream);
// fp32 -> bf16 (round to nearest even) of n elements
cudaError_t launch_f32_to_bf16(const float *src, int64_t n, void *dst, cudaStream_t stream);
// MX activations, the tensor-core scale layout and the block-scaled product
int64_t mx_padded_rows(int64_t R);
cudaError_t launch_mxfp8_quant(const void *X, int64_t M, int64_t K, uint8_t *codes, uint8_t *scales, int layout,
                               cudaStream_t stream);
cudaError_t launch_mx_scale_layout(const uint8_t *src, int64_t R, int64_t K, uint8_t *dst, cudaStream_t stream);
cudaError_t launch_mx_gemm(const uint8_t *x_codes, const uint8_t *x_sf, int64_t M, int64_t N, int64_t K,
                           const uint8_t *w_codes, const uint8_t *w_sf, void *Y, bool weights_static,
                           cudaStream_t stream);
size_t tc_workspace_bytes(int64_t M, int64_t N, int64_t K);
// byte range of the split-K tile counters inside that workspace (0 bytes if none)
void tc_workspace_counters(int64_t M, int64_t N, int64_t K, size_t *offset, size_t *bytes);
cudaError_t launch_gemm_tc(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                           const void *scales, const uint32_t *qzeros, int group, int mode, bool y_f32, void *Y,
                           void *ws, cudaStream_t stream);
size_t awq_workspace_bytes(int64_t M, int64_t N, int64_t K, int group, int mode, int n_alpha);
cudaError_t launch_awq_search(const void *W, const void *X, int64_t N, int64_t K, int64_t M, int group, int mode,
                              int n_alpha, double *losses, int *best, float *s_best, void *ws, cudaStream_t stream);
int read_and_clear_device_error();
// Time after which a kernel's wait for a copy, an MMA or another warp gives up
// (default kDefaultWaitNs; lowered only by tests of the failure path through
// w4_set_wait_limit_ns).  Waits that drain copies before a CTA exits always
// keep the default.
constexpr uint64_t kDefaultWaitNs = 200000000ull;   // 200 ms; no legitimate wait comes near it
// The kernels receive the limit in the low 63 bits of a launch parameter; the
// top bit, set only by w4_test_stall_first_wait, makes each warp's first wait
// for a copy target a barrier that nothing completes, so that it runs out.
constexpr uint64_t kStallFirstWait = 1ull << 63;
uint64_t wait_limit_ns();
__host__ __device__ inline uint64_t wait_limit_of(uint64_t w) { return w & ~kStallFirstWait; }
__host__ __device__ inline bool stalls_first_wait(uint64_t w) { return (w & kStallFirstWait) != 0; }
// Device address of the library's error word on the current device (nullptr on failure).
int *device_error_word();

}  // namespace w4
