// w4a16_gemm, M > 16: the tensor-core path (tcgen05, tensor memory, TMA).
//
// Method: page 4 (llm-glossary.tokens-kit.com/terms/quantization-methods/, GPTQ
// section) notes that large prefill GEMMs are governed by the dequantize /
// tensor-core path; page 3 (blog.freezetheflame.cc quantization deep dive)
// section 1.2 fuses dequantization into the GEMM so weights stay 4-bit in
// HBM, and its section 3.1 sketches Marlin (INT4 unpacked in registers, fed to
// tensor cores).  Dequantization follows page 5 (ai-infra.cypggs.com
// .../02-core-ideas) section 2.2, x^ = (q - zp) * s, rounded once to bf16.
//
// B200 design.  The MMA computes the transposed tile
//     D[128 channels, BN tokens] += W^[128 channels, 16 k] . X[BN tokens, 16 k]^T
// with tcgen05.mma kind::f16 (bf16 in, fp32 accumulate):
//   * A = the dequantized weights, written by the dequantizing warps straight
//     into TENSOR MEMORY with tcgen05.st (lane = output channel, 32-bit column
//     c of a stage = the bf16 pair (2c, 2c+1) of a 64-wide k-block).  The
//     weights never touch shared memory, which leaves the shared-memory
//     bandwidth to the activation operand;
//   * B = the activations, a [BN tokens x 64 k] bf16 box per k-block, brought
//     into shared memory by TMA with the 128-byte swizzle the UMMA descriptor
//     expects (K-major, 8-row atoms of 1024 bytes);
//   * D lives in tensor memory (BN fp32 columns); the epilogue reads it with
//     tcgen05.ld, one channel per lane, so a warp writes 32 consecutive
//     channels of one token (64 contiguous bytes of Y).
// Warp roles (320 threads): warp 0 issues the TMA loads, warp 1 allocates
// tensor memory and one of its threads issues the MMAs, warps 2..9 dequantize
// (warp w owns the 32 lanes 32*(w%4).. of tensor memory and every other
// k-block) and then run the epilogue.  A 4- or 6-stage ring couples them with
// mbarriers: full_b (TMA bytes landed), full_a (4 warps stored their A
// slice), empty (tcgen05.commit: the MMAs that read the stage are done).
// tcgen05.mma issue blocks until the previous MMA is nearly done, so the
// issuer never checks a barrier between two k-blocks on its own: the
// non-blocking tests of the next k-block's barriers go in the same block of
// PTX as the current k-block's MMAs, and their latency overlaps the MMAs.
// For the same reason the dequantizing loop is kept lean: two dequantizing
// warps share the issuer's sub-partition (tensor-memory lane quarters follow
// the warp index), and every instruction they issue can delay the next MMA.
// Every wait is bounded in time; a wait that runs out records an error code
// (read by w4_device_error), raises a CTA-wide abort flag, and the CTA drains
// its own in-flight copies and MMAs, frees its tensor memory and returns.
//
// Split-K: when the tile grid is too small for 148 SMs the k-blocks are split
// across CTAs; each writes an fp32 partial tile to the caller's workspace and
// the last CTA of a tile (found with an atomic counter) sums the partials in
// split order, writes Y and re-zeroes the counter.
#include "common.cuh"
#include "tc_ptx.cuh"

#include <cuda.h>

namespace w4 {

static __device__ int g_device_error;

namespace {

constexpr int kThreads = 320;
constexpr int kKB = 64;                      // k per block (one 128-byte swizzle row of bf16)

enum : int {
    kErrWaitTma = 0x101, kErrWaitFullA = 0x102, kErrWaitEmptyTma = 0x103, kErrWaitEmptyDeq = 0x104,
    kErrWaitDone = 0x105, kErrDrain = 0x106
};

// ---------------------------------------------------------------- PTX ----
// Wait for the phase of `bar` with the given parity.  Gives up (returns false)
// when the CTA's abort flag is raised or after `limit` ns, in which case it
// records `code` and raises the abort flag.
__device__ __noinline__ bool wait_bounded(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int code,
                                         uint64_t limit)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit) {
            *abort_flag = 1;
            atomicCAS(&g_device_error, 0, code);
            return false;
        }
    }
}

// Drain wait: ignores the abort flag, bounded in time only.
__device__ __noinline__ bool wait_drain(uint64_t *bar, uint32_t parity)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kDefaultWaitNs) {
            atomicCAS(&g_device_error, 0, kErrDrain);
            return false;
        }
    }
    return true;
}

// Bounded wait until both barriers have completed the phase with the given
// parity; each round tests both at once (their latencies overlap).
__device__ __noinline__ bool wait_pair_bounded(uint64_t *a, uint64_t *b, uint32_t parity, volatile int *abort_flag,
                                              uint64_t limit)
{
    const uint64_t t0 = globaltimer();
    while (true) {
        const bool ra = mbar_test(a, parity), rb = mbar_test(b, parity);
        if (ra && rb) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit) {
            *abort_flag = 1;
            atomicCAS(&g_device_error, 0, kErrWaitFullA);
            return false;
        }
    }
}

// One k-block (four 128 x BN x 16 MMAs, A from tensor memory at a_tmem, B
// from the SW128 descriptor bdesc, accumulate unless acc0 == 0 for the first)
// and its commit to `empty`, with non-blocking tests of the next k-block's
// barriers issued first; returns whether both were complete.
__device__ __forceinline__ bool mma_kblock_test_next(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc, uint32_t idesc,
                                                     uint32_t acc0, uint64_t *empty, uint64_t *next_a,
                                                     uint64_t *next_b, uint32_t next_parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred pa, pb, p0, p1;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 pa, [%1], %3;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 pb, [%2], %3;\n\t"
        "setp.ne.b32 p0, %8, 0;\n\t"
        "setp.eq.b32 p1, %8, %8;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%4], [%5], %6, %7, p0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%4], [%9], %10, %7, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%4], [%11], %12, %7, p1;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%4], [%13], %14, %7, p1;\n\t"
        "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%15];\n\t"
        "and.pred pa, pa, pb;\n\t"
        "selp.u32 %0, 1, 0, pa;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(next_a)), "r"(smem_u32(next_b)), "r"(next_parity), "r"(d_tmem), "r"(a_tmem), "l"(bdesc),
          "r"(idesc), "r"(acc0), "r"(a_tmem + 8), "l"(bdesc + 2), "r"(a_tmem + 16), "l"(bdesc + 4), "r"(a_tmem + 24),
          "l"(bdesc + 6), "r"(smem_u32(empty))
        : "memory");
    return ok != 0;
}

template <int BN>
struct TcCfg {
    static constexpr int kCols = (BN <= 128) ? 256 : 512;               // tensor-memory allocation
    // pipeline depth: as many 32-column A stages as fit beside the accumulator, at most 6 (even)
    static constexpr int kStages = ((kCols - BN) / 32 >= 6) ? 6 : 4;
    static constexpr int kACol0 = BN;                                   // A stages follow the BN fp32 accumulator columns
    static constexpr int kBBytes = BN * 128;                            // activation box bytes
    static constexpr int kCodeBytes = 128 * 32;                         // codes box: 128 channels x 64 k
    static constexpr int kStageBytes = kBBytes + kCodeBytes;            // a multiple of 1024
    static_assert(kACol0 + kStages * 32 <= kCols, "tensor memory overflow");
    static constexpr int kMinBlocks = (BN == 256) ? 1 : 2;
    // kind::f16, fp32 D, bf16 A and B, both K-major, N = BN, M = 128
    static constexpr uint32_t kIdesc =
        (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(128 >> 4) << 24);
};

// Scales and zero-points of one channel's two 32-weight halves of a k-block.
struct SlotData {
    unsigned short s0, s1;
    uint32_t z0, z1;
};

template <int BN>
__global__ void __launch_bounds__(kThreads, TcCfg<BN>::kMinBlocks)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_q,
               const __grid_constant__ CUtensorMap tmap_y, int y_tma, int M, int N, int K, int group_log2, int asym,
               const uint4 *__restrict__ qweight, const unsigned short *__restrict__ scales,
               const uint32_t *__restrict__ qzeros, void *__restrict__ Y, int y_f32, float *__restrict__ partial,
               unsigned *__restrict__ counters, int splits, int kb_per_split, uint64_t wait_ns)
{
    using C = TcCfg<BN>;
    constexpr int kStages = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    // (an offset from the shared array, not an integer cast, so that the
    // compiler keeps the shared address space and emits shared loads/stores)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint8_t *sB = smem;                                               // kStages x BN x 128 bytes
    uint64_t *full_b = (uint64_t *)(smem + kStages * C::kStageBytes);
    uint64_t *full_a = full_b + kStages;
    uint64_t *empty = full_a + kStages;
    uint64_t *done = empty + kStages;
    uint32_t *tmem_slot = (uint32_t *)(done + 1);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    int *last_flag = (int *)(tmem_slot + 2);
    uint64_t *stall = (uint64_t *)(tmem_slot + 4);      // a barrier nothing completes (failure tests)
    const uint64_t limit = wait_limit_of(wait_ns);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * 128, m0 = blockIdx.y * BN, split = blockIdx.z;
    const int KQ = K >> 5;                                            // 16-byte code chunks per channel
    const int kb_total = (K + kKB - 1) / kKB;
    const int kb_begin = split * kb_per_split;
    const int nkb = min(kb_total, kb_begin + kb_per_split) - kb_begin;
    const int NG = K >> group_log2, ZW = (NG + 7) >> 3;

    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; ++s) {
            mbar_init(&full_b[s], 1);
            mbar_init(&full_a[s], 4);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        mbar_init(stall, 1);
        *abort_flag = 0;
        *last_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::kCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;
    pdl_wait();                                                       // the previous kernel's writes are visible
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ TMA producer --
        if (lane == 0) {
            asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_x) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_q) : "memory");
            int issued = 0;
            for (int i = 0; i < nkb; ++i) {
                const int s = i % kStages;
                const uint32_t ph = (i / kStages) & 1;
                if (!mbar_try_wait(&empty[s], ph ^ 1) && !wait_bounded(&empty[s], ph ^ 1, abort_flag, kErrWaitEmptyTma, limit))
                    break;
                mbar_arrive_expect_tx(&full_b[s], C::kStageBytes);
                tma_load_2d(sB + s * C::kStageBytes, &tmap_x, &full_b[s], (kb_begin + i) * kKB, m0);
                tma_load_2d(sB + s * C::kStageBytes + C::kBBytes, &tmap_q, &full_b[s], (kb_begin + i) * 8, n0);
                ++issued;
            }
            // drain: every issued copy must have landed before the CTA may exit
            for (int i = max(0, issued - kStages); i < issued; ++i)
                wait_drain(&full_b[i % kStages], (i / kStages) & 1);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            // Per k-block: the four MMAs and the commit are issued in one
            // block of PTX together with non-blocking tests of the NEXT
            // k-block's two barriers, whose shared-memory latency (hundreds of
            // cycles under load) then overlaps the MMA issue instead of
            // leaving the tensor pipe idle (tcgen05.mma issue blocks until the
            // previous MMA is nearly done, so the issuer has no slack).
            // The loop is unrolled over the ring's stages, so that the stage,
            // its descriptor offset and its barriers are constants: between two
            // k-blocks the issuer runs only a handful of instructions.
            bool ready = false, stop = false;
            uint32_t ph = 0;
            const uint64_t bdesc0 = desc_k_sw128(smem_u32(sB));
            const uint32_t a0 = tmem + C::kACol0;
            for (int i0 = 0; i0 < nkb && !stop; i0 += kStages, ph ^= 1u) {
#pragma unroll
                for (int st = 0; st < kStages; ++st) {
                    const int i = i0 + st;
                    if (i >= nkb) break;
                    if (!ready) ready = wait_pair_bounded(&full_a[st], &full_b[st], ph, abort_flag, limit);
                    if (!ready) {
                        stop = true;
                        break;
                    }
                    tc_fence_after();
                    // the next k-block's stage and phase (the last k-block re-tests its own, complete, barriers)
                    const int s1 = (st + 1 == kStages) ? 0 : st + 1;
                    const uint32_t ph1 = (st + 1 == kStages) ? (ph ^ 1u) : ph;
                    const bool last = i + 1 == nkb;
                    ready = mma_kblock_test_next(tmem, a0 + st * 32,
                                                 bdesc0 + (uint64_t)((st * C::kStageBytes) >> 4), C::kIdesc,
                                                 i > 0 ? 1u : 0u, &empty[st], last ? &full_a[st] : &full_a[s1],
                                                 last ? &full_b[st] : &full_b[s1], last ? ph : ph1);
                }
            }
            mma_commit(done);
            wait_drain(done, 0);   // no MMA may still be running when tensor memory is freed
        }
        __syncwarp();
    } else {
        // ------------------------------------- dequantize, then epilogue --
        const int q = warp & 3;                      // tensor-memory lane quarter of this warp
        const int h = (warp - 2) >> 2;               // k-block parity handled by this warp
        const int r = 32 * q + lane;
        const int n = n0 + r;
        const bool okn = n < N;
        const unsigned short *srow = scales + (size_t)(okn ? n : 0) * NG;
        const uint32_t *zrow = qzeros + (size_t)(okn ? n : 0) * ZW;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);

        // the codes arrive with the activations (TMA, full_b); only the scales
        // and zero-points are loaded here, D k-blocks of this warp ahead
        uint32_t magic;                              // 0x43004300, opaque to the compiler
        asm volatile("mov.b32 %0, 0x43004300;" : "=r"(magic));
        constexpr int D = 4;
        SlotData buf[D];
        auto fetch = [&](int i, SlotData &sd) {
            const int kq = (kb_begin + i) * 2;       // first 32-weight half of this k-block
            const bool ok0 = okn && kq < KQ, ok1 = okn && (kq + 1 < KQ);
            const int j0 = (kq * 32) >> group_log2, j1 = ((kq + 1) * 32) >> group_log2;
            // (with g >= 64 both halves of a k-block lie in one group: j1 == j0)
            sd.s0 = ok0 ? __ldg(srow + j0) : (unsigned short)0;
            sd.z0 = !asym ? 8u : ok0 ? (__ldg(zrow + (j0 >> 3)) >> (4 * (j0 & 7))) & 0xFu : 0u;
            if (group_log2 == 5) {
                sd.s1 = ok1 ? __ldg(srow + j1) : (unsigned short)0;
                sd.z1 = !asym ? 8u : ok1 ? (__ldg(zrow + (j1 >> 3)) >> (4 * (j1 & 7))) & 0xFu : 0u;
            } else {
                sd.s1 = ok1 ? sd.s0 : (unsigned short)0;
                sd.z1 = ok1 ? sd.z0 : 0u;
            }
        };
#pragma unroll
        for (int d = 0; d < D; ++d)
            if (h + 2 * d < nkb) fetch(h + 2 * d, buf[d]);

        bool ok = true;
        int s = h;                                   // stage and phase of k-block i (i = h, h + 2, ...; kStages is even)
        uint32_t ph = 0;
        static_assert(kStages % 2 == 0, "the dequantizing warps step two stages at a time");
        for (int i0 = h; i0 < nkb && ok; i0 += 2 * D) {
#pragma unroll
            for (int d = 0; d < D; ++d) {
                const int i = i0 + 2 * d;
                if (i >= nkb || !ok) break;
                // full_b also means the MMAs of this stage's previous round are done
                // (the producer refilled it only after their commit), so its
                // tensor-memory A columns are free
                // (the inline try_wait is the usual case: the stage landed long ago)
                // (the first wait of a dequantizing warp targets a barrier that
                // nothing completes in the failure-path tests)
                uint64_t *fb = (i == h && stalls_first_wait(wait_ns)) ? stall : &full_b[s];
                const uint32_t fph = fb == stall ? 0u : ph;
                if (!__all_sync(0xffffffffu, mbar_try_wait(fb, fph) ||
                                                 wait_bounded(fb, fph, abort_flag, kErrWaitEmptyDeq, limit))) {
                    ok = false;
                    break;
                }
                // this channel's 64 codes: 32 bytes of row r of the codes box
                const uint4 *cs = (const uint4 *)(sB + s * C::kStageBytes + C::kBBytes + r * 32);
                const uint4 w0 = cs[0], w1 = cs[1];
                uint32_t v[32];
                const GroupConst c0 = group_const(buf[d].s0, buf[d].z0);
                GroupConst c1 = c0;
                if (group_log2 == 5 || buf[d].s1 != buf[d].s0 || buf[d].z1 != buf[d].z0)
                    c1 = group_const(buf[d].s1, buf[d].z1);
                if (i + 2 * D < nkb) fetch(i + 2 * D, buf[d]);
                const uint32_t wa[4] = {w0.x, w0.y, w0.z, w0.w};
                const uint32_t wb[4] = {w1.x, w1.y, w1.z, w1.w};
#pragma unroll
                for (int w = 0; w < 4; ++w)
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        v[4 * w + j] = dequant_pair(wa[w], j, c0, magic);
                        v[16 + 4 * w + j] = dequant_pair(wb[w], j, c1, magic);
                    }
                tmem_st32(lane_addr + C::kACol0 + s * 32, v);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&full_a[s]);
                s += 2;
                if (s >= kStages) {
                    s -= kStages;
                    ph ^= 1u;
                }
            }
        }

        // ---- epilogue: accumulator -> Y (or fp32 partials) ----
        const bool have = __all_sync(0xffffffffu, ok && wait_bounded(done, 0, abort_flag, kErrWaitDone, limit));
        tc_fence_after();
        constexpr int HALF = BN / 2;                  // columns per warp of a lane quarter
        const int cbeg = h * HALF;
        if (have && y_tma) {
            // bf16 tile [BN tokens][128 channels] in the (now idle) stage buffers,
            // stored below by one TMA: every warp store writes 64 contiguous bytes
            __nv_bfloat16 *ysm = (__nv_bfloat16 *)smem;
            constexpr int CH = HALF < 64 ? HALF : 64;
            for (int c = 0; c < HALF; c += CH) {
                float acc[CH];
                if (CH >= 32) {
#pragma unroll
                    for (int u = 0; u < CH / 32; ++u) tmem_ld32(lane_addr + cbeg + c + 32 * u, acc + 32 * u);
                } else {
#pragma unroll
                    for (int u = 0; u < CH / 8; ++u) tmem_ld8(lane_addr + cbeg + c + 8 * u, acc + 8 * u);
                }
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < CH; ++j) ysm[(cbeg + c + j) * 128 + r] = __float2bfloat16_rn(acc[j]);
            }
        } else if (have) {
            // columns in chunks of CH (64, or the whole half when it is smaller),
            // all loads of a chunk issued before one wait
            constexpr int CH = HALF < 64 ? HALF : 64;
            for (int c = 0; c < HALF; c += CH) {
                float acc[CH];
                if (CH >= 32) {
#pragma unroll
                    for (int u = 0; u < CH / 32; ++u) tmem_ld32(lane_addr + cbeg + c + 32 * u, acc + 32 * u);
                } else {
#pragma unroll
                    for (int u = 0; u < CH / 8; ++u) tmem_ld8(lane_addr + cbeg + c + 8 * u, acc + 8 * u);
                }
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    const int m = m0 + cbeg + c + j;
                    if (okn && m < M) {
                        if (splits == 1) store_y(Y, (size_t)m * N + n, acc[j], y_f32);
                        else partial[((size_t)split * M + m) * N + n] = acc[j];
                    }
                }
            }
        }
        if (y_tma) {
            // make the tile visible to the TMA unit, then one thread stores it
            // (rows past M and channels past N are clipped) and waits until
            // shared memory has been read
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (threadIdx.x == 64 && *abort_flag == 0) {
                asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];" ::"l"(
                                 &tmap_y),
                             "r"(smem_u32(smem)), "r"(n0), "r"(m0)
                             : "memory");
                asm volatile("cp.async.bulk.commit_group;" ::: "memory");
                asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
            }
        }
        if (splits > 1) {
            __threadfence();
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (threadIdx.x == 64) {
                const unsigned tile = blockIdx.y * gridDim.x + blockIdx.x;
                const unsigned prev = atomicAdd(&counters[tile], 1u);
                *last_flag = (prev == (unsigned)splits - 1) ? 1 : 0;
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            if (*(volatile int *)last_flag) {
                __threadfence();
                for (int c = 0; c < HALF; ++c) {
                    const int m = m0 + cbeg + c;
                    if (okn && m < M) {
                        float sum = 0.f;
                        for (int sp = 0; sp < splits; ++sp) sum += __ldcg(partial + ((size_t)sp * M + m) * N + n);
                        store_y(Y, (size_t)m * N + n, sum, y_f32);
                    }
                }
                if (threadIdx.x == 64) counters[blockIdx.y * gridDim.x + blockIdx.x] = 0u;
            }
        }
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kCols);
}

// ----------------------------------------------------------------- host --


struct TcPlan {
    int BN = 0, splits = 1, kb_per_split = 0, m_tiles = 0, n_tiles = 0;
    size_t ws_bytes = 0;
};

int pick_bn(int64_t M)
{
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

TcPlan plan_tc(int64_t M, int64_t N, int64_t K)
{
    TcPlan p;
    p.BN = pick_bn(M);
    p.m_tiles = (int)((M + p.BN - 1) / p.BN);
    p.n_tiles = (int)((N + 127) / 128);
    const int kb_total = (int)((K + kKB - 1) / kKB);
    const int64_t tiles = (int64_t)p.m_tiles * p.n_tiles;
    const int per_sm = (p.BN == 256) ? 1 : 2;
    const int64_t slots = (int64_t)kNumSMs * per_sm;
    int best = 1;
    if (p.BN <= 64 && tiles < 4 * slots) {
        // skinny, bandwidth-bound: split k so the grid fills whole waves of the SMs
        double best_eff = -1.0;
        for (int s = 1; s <= 8 && kb_total / s >= 4; ++s) {
            const int64_t ctas = tiles * s;
            const int64_t waves = (ctas + slots - 1) / slots;
            const double eff = (double)ctas / (double)(waves * slots);
            if (eff > best_eff + 0.02) { best_eff = eff; best = s; }
        }
    }
    p.kb_per_split = (kb_total + best - 1) / best;
    p.splits = (kb_total + p.kb_per_split - 1) / p.kb_per_split;
    if (p.splits > 1) {
        const size_t part = (size_t)p.splits * M * N * sizeof(float);
        const size_t part_al = (part + 255) & ~(size_t)255;
        p.ws_bytes = part_al + (size_t)tiles * sizeof(unsigned);
    }
    return p;
}

template <int BN>
cudaError_t launch_bn(const CUtensorMap &map, const CUtensorMap &qmap, const CUtensorMap &ymap, int y_tma,
                      const TcPlan &p, int M, int N, int K, int glog2, int asym,
                      const uint32_t *qweight, const void *scales, const uint32_t *qzeros, void *Y, int y_f32,
                      void *ws, cudaStream_t stream)
{
    using C = TcCfg<BN>;
    size_t smem = 1024 + C::kStages * C::kStageBytes + 256;
    if (C::kMinBlocks == 2 && smem < 80 * 1024) smem = 80 * 1024;   // at most 2 CTAs share an SM's tensor memory
    static std::atomic<bool> attr_done[kMaxDevices];   // the attribute is per device
    {
        const cudaError_t e = set_smem_attr(gemm_tc_kernel<BN>, (int)smem, attr_done);
        if (e != cudaSuccess) return e;
    }
    float *partial = nullptr;
    unsigned *counters = nullptr;
    if (p.splits > 1) {
        const size_t part = (size_t)p.splits * M * N * sizeof(float);
        partial = (float *)ws;
        counters = (unsigned *)((uint8_t *)ws + ((part + 255) & ~(size_t)255));
    }
    dim3 grid(p.n_tiles, p.m_tiles, p.splits);
    return launch_pdl(gemm_tc_kernel<BN>, grid, dim3(kThreads), smem, stream, map, qmap, ymap, y_tma, M, N, K, glog2,
                      asym, (const uint4 *)qweight, (const unsigned short *)scales, qzeros, Y, y_f32,
                      partial, counters, p.splits, p.kb_per_split, wait_limit_ns());
}

}  // namespace

size_t tc_workspace_bytes(int64_t M, int64_t N, int64_t K) { return plan_tc(M, N, K).ws_bytes; }

void tc_workspace_counters(int64_t M, int64_t N, int64_t K, size_t *offset, size_t *bytes)
{
    const TcPlan p = plan_tc(M, N, K);
    *offset = 0;
    *bytes = 0;
    if (p.splits > 1) {
        const size_t part = (size_t)p.splits * M * N * sizeof(float);
        *offset = (part + 255) & ~(size_t)255;
        *bytes = p.ws_bytes - *offset;
    }
}

cudaError_t launch_gemm_tc(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                           const void *scales, const uint32_t *qzeros, int group, int mode, bool y_f32, void *Y,
                           void *ws, cudaStream_t stream)
{
    const TcPlan p = plan_tc(M, N, K);
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUtensorMap map;
    const cuuint64_t gdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t gstride[1] = {(cuuint64_t)K * 2};
    const cuuint32_t box[2] = {(cuuint32_t)kKB, (cuuint32_t)p.BN};
    const cuuint32_t estride[2] = {1, 1};
    const CUresult cr = enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(X), gdim, gstride, box,
                            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (cr != CUDA_SUCCESS) return cudaErrorInvalidValue;
    // the codes as 32-bit words [N][K/8]; one box = 128 channels x one 64-wide k-block
    CUtensorMap qmap;
    const cuuint64_t qdim[2] = {(cuuint64_t)(K / 8), (cuuint64_t)N};
    const cuuint64_t qstride[1] = {(cuuint64_t)K / 2};
    const cuuint32_t qbox[2] = {8u, 128u};
    if (enc(&qmap, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(qweight), qdim, qstride, qbox, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // Y tiles leave through one TMA store per CTA when Y's rows are 16-byte
    // aligned; otherwise (and for split-K partials) the epilogue stores directly
    CUtensorMap ymap = map;
    int y_tma = 0;
    if (!y_f32 && p.splits == 1 && ((uintptr_t)Y % 16) == 0 && (N * 2) % 16 == 0) {
        const cuuint64_t ydim[2] = {(cuuint64_t)N, (cuuint64_t)M};
        const cuuint64_t ystride[1] = {(cuuint64_t)N * 2};
        const cuuint32_t ybox[2] = {128u, (cuuint32_t)p.BN};
        if (enc(&ymap, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, Y, ydim, ystride, ybox, estride,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_NONE,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
        y_tma = 1;
    }
    const int glog2 = group == 32 ? 5 : group == 64 ? 6 : 7;
    const int asym = mode == W4_ASYM;
    switch (p.BN) {
    case 16: return launch_bn<16>(map, qmap, ymap, y_tma, p, (int)M, (int)N, (int)K, glog2, asym, qweight, scales, qzeros, Y, y_f32 ? 1 : 0, ws, stream);
    case 32: return launch_bn<32>(map, qmap, ymap, y_tma, p, (int)M, (int)N, (int)K, glog2, asym, qweight, scales, qzeros, Y, y_f32 ? 1 : 0, ws, stream);
    case 64: return launch_bn<64>(map, qmap, ymap, y_tma, p, (int)M, (int)N, (int)K, glog2, asym, qweight, scales, qzeros, Y, y_f32 ? 1 : 0, ws, stream);
    case 128: return launch_bn<128>(map, qmap, ymap, y_tma, p, (int)M, (int)N, (int)K, glog2, asym, qweight, scales, qzeros, Y, y_f32 ? 1 : 0, ws, stream);
    default: return launch_bn<256>(map, qmap, ymap, y_tma, p, (int)M, (int)N, (int)K, glog2, asym, qweight, scales, qzeros, Y, y_f32 ? 1 : 0, ws, stream);
    }
}

int *device_error_word()
{
    static int *addr[64] = {};                   // per device, resolved once
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
    if (!addr[dev]) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_device_error) != cudaSuccess) return nullptr;
        addr[dev] = (int *)p;
    }
    return addr[dev];
}

int read_and_clear_device_error()
{
    int v = 0;
    if (cudaMemcpyFromSymbol(&v, g_device_error, sizeof(int)) != cudaSuccess) return -1;
    const int zero = 0;
    if (v != 0 && cudaMemcpyToSymbol(g_device_error, &zero, sizeof(int)) != cudaSuccess) return -1;
    return v;
}

}  // namespace w4
