// w4a16_gemm, M <= 16: the decode GEMV / skinny path.
//
// Method: page 2 (learn.longtimenohack.com .../quantization.html) opens with
// "reading weights is the top cost of decode", page 4
// (llm-glossary.tokens-kit.com/terms/quantization-methods/, GPTQ section) with
// "small-batch decode profits from the weight bandwidth", and page 3
// (blog.freezetheflame.cc quantization deep dive) section 1.2 with "fuse
// dequantize into the GEMM so the weights stay 4-bit in HBM"; section 2.2 of
// the same page prefetches the group scales to shared memory, and its section
// 3.1 sketches Marlin, which unpacks INT4 in registers and feeds mma.sync.
// Dequantization follows page 5 (ai-infra.cypggs.com .../02-core-ideas)
// section 2.2, x^ = (q - zp) * s, rounded once to bf16.
//
// Design (HBM-bound: 0.5 B of codes + 1/64 B of scale per weight at g = 128;
// the dequantization costs about 2.5 issue slots per weight, which is close to
// the issue budget of the SMs at HBM speed, so the kernel must stream the codes
// without spending instructions on it):
//   * a CTA (4 warps, or 8 when there are fewer than two tiles per SM) owns a
//     tile of 16 output channels and all of K; warp w takes the 512-wide
//     k-stages w, w+W, w+2W, ... and the partial tiles are summed in shared
//     memory at the end (no global scratch);
//   * the codes stream HBM -> shared memory by TMA (one 2-D box of 16 rows x
//     128 bytes per k-box, 128-byte swizzle), four boxes in flight per warp on
//     the warp's own mbarrier ring, so a resident CTA keeps 32 KB of reads
//     outstanding and the loads cost the warps one instruction per box;
//   * per k-box, each lane turns one (channel, group) scale and zero-point into
//     the bf16x2 constants below and parks them in the warp's shared-memory
//     slot, where the lanes that need them read them back (the scales and
//     zero-points of the next box are loaded while this one is computed, and
//     the tile's whole scale and zero-point rows are asked into L2 at launch);
//   * lane (g, t) = (lane/4, lane%4) reads, for channels g and g+8, the 16-byte
//     chunks t and t+4 of the box (the swizzle makes these reads free of bank
//     conflicts) and the activations of the same k from global memory;
//   * each 32-bit word of codes gives four bf16x2 pairs of ADJACENT elements
//     with one shift and one LOP3 (the packed layout keeps even elements in
//     the low half-word), as 128 + u via the bf16 exponent of 128;
//   * exact w^ = bf16_rne((u - zp) * s16) with three bf16x2 operations:
//     D = (128+u) - (128+zp) (exact), c = D * s_lo (exact: <= 7 bits) and
//     w^ = fma(D, s_hi, c), where s16 = s_hi + s_lo splits the fp16 scale into
//     its bf16 rounding and the (<= 3-bit) remainder; the fused multiply-add
//     rounds the exact product D * s16 once;
//   * mma.sync m16n8k16 (bf16 in, fp32 accumulate) takes those registers as
//     its A fragment directly: the k-order inside an MMA is free, so a
//     thread's logical columns (2t, 2t+1) and (2t+8, 2t+9) are mapped to the
//     physical elements {0,1} and {2,3} (then {4,5} and {6,7}) of its own
//     words, and the activation fragment for token g is then the plain 16-byte
//     chunk of X[g] at the word's k;
//   * tokens occupy the MMA's N = 8 columns, MT groups of 8 tokens (M <= 8 * MT);
//     lanes whose token is >= M repeat token M-1 into MMA columns that are
//     never stored.
// Every wait on an mbarrier is bounded in time; a wait that runs out records
// an error code (read by w4_device_error), and the warp stops computing, waits
// (again bounded) for its own copies in flight and returns.
#include "common.cuh"

#include <cuda.h>

namespace w4 {
namespace {

constexpr int kBoxK = 256;                       // k per TMA box: 32 words of 8 codes
constexpr int kBoxBytes = 16 * 128;              // 16 channels x 128 bytes
constexpr int kBoxesPerStage = 2;                // a pipeline stage is two boxes: 512 k
constexpr int kStageK = kBoxK * kBoxesPerStage;
constexpr int kStageBytes = kBoxBytes * kBoxesPerStage;
constexpr int kStages = 2;                       // stages in flight per warp (8 KB)
constexpr uint64_t kWaitLimitNs = 200000000ull;  // 200 ms; a box lands in microseconds
constexpr int kErrGemvWait = 0x201, kErrGemvDrain = 0x202;

__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ uint64_t globaltimer()
{
    uint64_t t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity; false after kWaitLimitNs.
__device__ __noinline__ bool wait_box(uint32_t bar, uint32_t parity)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity))
        if (globaltimer() - t0 > kWaitLimitNs) return false;
    return true;
}

// a + b on bf16 pairs.  The dequantization adds -(128 + zp), negated once per
// group, because a subtraction of bf16 pairs costs an extra sign flip.
__device__ __forceinline__ uint32_t bf2_add(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("add.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bf2_mul(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("mul.rn.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bf2_fma(uint32_t a, uint32_t b, uint32_t c)
{
    uint32_t d;
    asm("fma.rn.bf16x2 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(c));
    return d;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Per-(channel, group) dequantization constants, each duplicated into both
// halves of a bf16x2: s_hi = bf16_rne(s16), s_lo = s16 - s_hi, and -Z = -(128 + zp).
__device__ __forceinline__ uint4 group_const(unsigned short s16bits, uint32_t zp)
{
    const float sf = __half2float(__ushort_as_half(s16bits));
    const __nv_bfloat16 hi = __float2bfloat16_rn(sf);
    const __nv_bfloat16 lo = __float2bfloat16_rn(sf - __bfloat162float(hi));   // exact
    const uint32_t h = __bfloat16_as_ushort(hi), l = __bfloat16_as_ushort(lo);
    return make_uint4(h | (h << 16), l | (l << 16), 0xC300C300u | (zp << 16) | zp, 0x43004300u);
}

// w^ for elements (2j, 2j+1) of packed word q.
__device__ __forceinline__ uint32_t dequant_pair(uint32_t q, int j, const uint4 &gc)
{
    // 128 + u as bf16x2: (q >> 4j) & 0x000F000F | 0x43004300 in one LOP3; the
    // constant 0x43004300 comes from shared memory (gc.w) so that it stays in a
    // register instead of costing a second LOP3 per pair
    uint32_t v;
    asm("lop3.b32 %0, %1, %2, %3, 0xEA;" : "=r"(v) : "r"(q >> (4 * j)), "r"(0x000F000Fu), "r"(gc.w));
    const uint32_t D = bf2_add(v, gc.z);
    return bf2_fma(D, gc.x, bf2_mul(D, gc.y));
}

// Dynamic shared-memory layout of one GEMV CTA.
template <int G, int MT, int kWarps>
struct GemvSmem {
    static constexpr int kConstOff = kWarps * kStages * kStageBytes;
    static constexpr int kRedOff = kConstOff + kWarps * 16 * (kStageK / G) * 16;
    static constexpr int kBarOff = kRedOff + kWarps * 32 * 4 * MT * 4;
    static constexpr int kBytes = kBarOff + kWarps * kStages * 8 + 1024;   // + alignment slack
};

template <int G, int MODE, int MT, int kWarps>
__global__ void __launch_bounds__(kWarps * 32, kWarps == 8 ? 2 : (MT == 1 ? 5 : 4))
gemv_kernel(const __grid_constant__ CUtensorMap tmap_q, const uint4 *__restrict__ X, int M, int N, int K,
            const unsigned short *__restrict__ scales, const uint32_t *__restrict__ qzeros,
            __nv_bfloat16 *__restrict__ Y, int *err)
{
    constexpr int GPB = kStageK / G;             // groups per stage and channel
    constexpr int CPL = 16 * GPB / 32;           // constants computed per lane and stage
    // dynamic shared memory: the stages (1024-byte aligned for the swizzle),
    // the constants, the cross-warp reduction and the barriers
    extern __shared__ uint8_t smem_raw[];
    using L = GemvSmem<G, MT, kWarps>;
    // (an offset from the shared array, not an integer cast, so that the
    // compiler keeps the shared address space and emits shared loads)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    auto sbox = (uint8_t(*)[kStages][kStageBytes])(smem);
    auto sconst = (uint4(*)[16 * GPB])(smem + L::kConstOff);
    auto red = (float(*)[32][4 * MT])(smem + L::kRedOff);
    auto full = (uint64_t(*)[kStages])(smem + L::kBarOff);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int NG = K / G, ZW = (NG + 7) >> 3;
    const int NS = (K + kStageK - 1) / kStageK;  // stages per channel
    const int nsw = (NS - warp + kWarps - 1) / kWarps;   // stages of this warp: warp, warp+4, ...
    const int r0 = (int)blockIdx.x * 16;

    const uint32_t bar0 = smem_u32(&full[warp][0]);
    const uint32_t box0 = smem_u32(&sbox[warp][0][0]);
    if (lane == 0) {
        for (int s = 0; s < kStages; ++s)
            asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8 * s));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_q) : "memory");
    }
    __syncwarp();
    pdl_wait();                                  // the previous kernel's writes are visible
    pdl_launch_dependents();
    auto issue = [&](int i) {                    // lane 0: stage i of this warp into slot i % kStages
        const int s = i % kStages;
        const int sb = warp + kWarps * i;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar0 + 8 * s),
                     "r"(kStageBytes)
                     : "memory");
#pragma unroll
        for (int bb = 0; bb < kBoxesPerStage; ++bb)   // a box past the end of K is zero-filled
            asm volatile(
                "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
                "[%2];" ::"r"(box0 + s * kStageBytes + bb * kBoxBytes),
                "l"(&tmap_q), "r"(bar0 + 8 * s), "r"((sb * kBoxesPerStage + bb) * 32), "r"(r0)
                : "memory");
    };
    if (lane == 0)
        for (int i = 0; i < kStages && i < nsw; ++i) issue(i);
    if (threadIdx.x == 32) {                     // the tile's scales and zero-points, HBM -> L2
        const int rows = min(16, N - r0);
        prefetch_l2(scales + (size_t)r0 * NG, (size_t)rows * NG * 2);
        if (MODE == W4_ASYM) prefetch_l2(qzeros + (size_t)r0 * ZW, (size_t)rows * ZW * 4);
    }

    // scales / zero-points of the constants this lane computes for stage i
    unsigned short sv[CPL];
    uint32_t zv[CPL];
    auto load_consts = [&](int i) {
        const int sb = warp + kWarps * i;
#pragma unroll
        for (int u = 0; u < CPL; ++u) {
            const int idx = lane + 32 * u, row = r0 + (idx & 15), j = sb * GPB + (idx >> 4);
            const bool ok = row < N && j < NG;
            sv[u] = ok ? __ldg(scales + (size_t)row * NG + j) : (unsigned short)0;
            if (MODE == W4_ASYM) zv[u] = ok ? (__ldg(qzeros + (size_t)row * ZW + (j >> 3)) >> (4 * (j & 7))) & 0xFu : 0u;
            else zv[u] = 8u;
        }
    };
    if (nsw > 0) load_consts(0);

    // two accumulator sets (the first and the second MMA of every word pair)
    // halve the dependent chain of MMAs
    float acc[MT][4], acc2[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][e] = acc2[mt][e] = 0.f;
    // a token past M reads token M-1: its MMA column is never stored
    const uint4 *xrows[MT];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) xrows[mt] = X + (size_t)min(g + 8 * mt, M - 1) * (K / 8);

    bool ok = true;
    int i = 0;
    for (; i < nsw; ++i) {
        const int sb = warp + kWarps * i;
        const int s = i % kStages;
        // constants of this stage into the warp's slot, then the next stage's loads
        __syncwarp();                            // every lane is done with the previous stage's slot
#pragma unroll
        for (int u = 0; u < CPL; ++u) sconst[warp][lane + 32 * u] = group_const(sv[u], zv[u]);
        if (i + 1 < nsw) load_consts(i + 1);
        __syncwarp();
        if (!wait_box(bar0 + 8 * s, (uint32_t)(i / kStages) & 1u)) {
            ok = false;
            break;
        }
        const uint8_t *st = &sbox[warp][s][0];
#pragma unroll
        for (int h = 0; h < 2 * kBoxesPerStage; ++h) {
            const int bb = h >> 1;               // box of this chunk
            const int c = t + 4 * (h & 1);       // chunk of the box (16 bytes of a 128-byte row)
            // this lane's codes: channels g and g+8, chunk c (128-byte swizzle)
            const uint4 wa4 = *(const uint4 *)(st + bb * kBoxBytes + g * 128 + ((c ^ g) << 4));
            const uint4 wb4 = *(const uint4 *)(st + bb * kBoxBytes + (g + 8) * 128 + ((c ^ g) << 4));
            // first k of the chunk; a chunk past the end of K (K is a multiple of
            // 32, chunks are whole) reads the last chunk's activations instead:
            // its codes are zero-filled by TMA and its groups' constants have
            // s16 = 0, so every w^ there is 0 and the activations only need to
            // be finite
            const int k0 = min(sb * kStageK + bb * kBoxK + c * 32, K - 32);
            const int gl = (bb * kBoxK + c * 32) / G;     // group of the chunk within the stage
            const uint4 ca = sconst[warp][g + 16 * gl];
            const uint4 cb = sconst[warp][(g + 8) + 16 * gl];
            const uint32_t wa[4] = {wa4.x, wa4.y, wa4.z, wa4.w};
            const uint32_t wb[4] = {wb4.x, wb4.y, wb4.z, wb4.w};
            uint4 xv[MT][4];
#pragma unroll
            for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                for (int w = 0; w < 4; ++w) xv[mt][w] = __ldg(xrows[mt] + k0 / 8 + w);
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t a0 = dequant_pair(wa[w], 0, ca), a1 = dequant_pair(wa[w], 1, ca);
                const uint32_t a2 = dequant_pair(wa[w], 2, ca), a3 = dequant_pair(wa[w], 3, ca);
                const uint32_t b0 = dequant_pair(wb[w], 0, cb), b1 = dequant_pair(wb[w], 1, cb);
                const uint32_t b2 = dequant_pair(wb[w], 2, cb), b3 = dequant_pair(wb[w], 3, cb);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    mma_bf16_16816(acc[mt], a0, b0, a1, b1, xv[mt][w].x, xv[mt][w].y);
                    mma_bf16_16816(acc2[mt], a2, b2, a3, b3, xv[mt][w].z, xv[mt][w].w);
                }
            }
        }
        __syncwarp();                            // the stage is read: refill it
        if (lane == 0 && i + kStages < nsw) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(i + kStages);
        }
    }
    if (!ok) {
        // a box never landed: record it, wait (bounded) for the copies this warp
        // still has in flight, and leave the tile unwritten
        if (lane == 0) {
            atomicCAS(err, 0, kErrGemvWait);
            for (int j = i; j < nsw && j < i + kStages; ++j)
                if (!wait_box(bar0 + 8 * (j % kStages), (uint32_t)(j / kStages) & 1u)) atomicCAS(err, 0, kErrGemvDrain);
        }
    }

#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) red[warp][lane][4 * mt + e] = acc[mt][e] + acc2[mt][e];
    const int all_ok = __syncthreads_and(ok ? 1 : 0);
    if (warp == 0 && all_ok) {
        const int rA = r0 + g, rB = rA + 8;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int w = 0; w < kWarps; ++w)
#pragma unroll
                for (int e = 0; e < 4; ++e) sm[e] += red[w][lane][4 * mt + e];
            const int m0 = 8 * mt + 2 * t, m1 = m0 + 1;   // tokens of c0/c2 and c1/c3
            if (rA < N && m0 < M) Y[(size_t)m0 * N + rA] = __float2bfloat16_rn(sm[0]);
            if (rA < N && m1 < M) Y[(size_t)m1 * N + rA] = __float2bfloat16_rn(sm[1]);
            if (rB < N && m0 < M) Y[(size_t)m0 * N + rB] = __float2bfloat16_rn(sm[2]);
            if (rB < N && m1 < M) Y[(size_t)m1 * N + rB] = __float2bfloat16_rn(sm[3]);
        }
    }
}

typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = (EncodeTiledFn)p;
    }
    return fn;
}

template <int G, int MODE, int MT, int W>
cudaError_t launch_gw(const CUtensorMap &map, const void *X, int64_t M, int64_t N, int64_t K, const void *scales,
                      const uint32_t *qzeros, void *Y, int *err, cudaStream_t stream)
{
    const int64_t blocks = (N + 15) / 16;       // one 16-channel tile per CTA
    constexpr int smem = GemvSmem<G, MT, W>::kBytes;
    static bool attr_set = false;
    if (!attr_set) {
        const cudaError_t e = cudaFuncSetAttribute(gemv_kernel<G, MODE, MT, W>,
                                                   cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess) return e;
        attr_set = true;
    }
    return launch_pdl(gemv_kernel<G, MODE, MT, W>, dim3((unsigned)blocks), dim3(W * 32), smem, stream, map,
                      (const uint4 *)X, (int)M, (int)N, (int)K, (const unsigned short *)scales, qzeros,
                      (__nv_bfloat16 *)Y, err);
}

// Few tiles (fewer than two per SM) get 8 warps each, so that the SMs still
// hold enough warps to hide latency; otherwise 4 warps per tile.
template <int G, int MODE, int MT>
cudaError_t launch_g(const CUtensorMap &map, const void *X, int64_t M, int64_t N, int64_t K, const void *scales,
                     const uint32_t *qzeros, void *Y, int *err, cudaStream_t stream)
{
    if ((N + 15) / 16 <= 2 * kNumSMs)
        return launch_gw<G, MODE, MT, 8>(map, X, M, N, K, scales, qzeros, Y, err, stream);
    return launch_gw<G, MODE, MT, 4>(map, X, M, N, K, scales, qzeros, Y, err, stream);
}

template <int MT>
cudaError_t launch_mt(const CUtensorMap &map, const void *X, int64_t M, int64_t N, int64_t K, const void *scales,
                      const uint32_t *qzeros, int group, int mode, void *Y, int *err, cudaStream_t stream)
{
    switch (group * 2 + mode) {
    case 32 * 2 + W4_SYM: return launch_g<32, W4_SYM, MT>(map, X, M, N, K, scales, qzeros, Y, err, stream);
    case 32 * 2 + W4_ASYM: return launch_g<32, W4_ASYM, MT>(map, X, M, N, K, scales, qzeros, Y, err, stream);
    case 64 * 2 + W4_SYM: return launch_g<64, W4_SYM, MT>(map, X, M, N, K, scales, qzeros, Y, err, stream);
    case 64 * 2 + W4_ASYM: return launch_g<64, W4_ASYM, MT>(map, X, M, N, K, scales, qzeros, Y, err, stream);
    case 128 * 2 + W4_SYM: return launch_g<128, W4_SYM, MT>(map, X, M, N, K, scales, qzeros, Y, err, stream);
    case 128 * 2 + W4_ASYM: return launch_g<128, W4_ASYM, MT>(map, X, M, N, K, scales, qzeros, Y, err, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

cudaError_t launch_gemv(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                        const void *scales, const uint32_t *qzeros, int group, int mode, void *Y,
                        cudaStream_t stream)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    int *err = device_error_word();
    if (!err) return cudaErrorUnknown;
    // the codes as a 2-D array of 32-bit words [N][K/8]; one box = 16 channels x 32 words
    CUtensorMap map;
    const cuuint64_t gdim[2] = {(cuuint64_t)(K / 8), (cuuint64_t)N};
    const cuuint64_t gstride[1] = {(cuuint64_t)K / 2};
    const cuuint32_t box[2] = {32u, 16u};
    const cuuint32_t estride[2] = {1u, 1u};
    const CUresult cr = enc(&map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(qweight), gdim, gstride,
                            box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
    if (M <= 8) return launch_mt<1>(map, X, M, N, K, scales, qzeros, group, mode, Y, err, stream);
    return launch_mt<2>(map, X, M, N, K, scales, qzeros, group, mode, Y, err, stream);
}

}  // namespace w4
