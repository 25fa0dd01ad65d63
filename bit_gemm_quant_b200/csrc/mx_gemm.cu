// w4_mx_gemm: Y = X^ . W^^T for MXFP8 activations and MXFP4 weights on the
// block-scaled tensor cores (tcgen05.mma kind::mxf8f6f4).
//
// Method: page 3 (blog.freezetheflame.cc quantization deep dive) section 4.3:
// FP4 weights packed two per byte, activations kept at FP8, one E8M0 scale per
// 32-element block, and an FP4 x FP8 tensor-core instruction accumulating at
// higher precision; page 2 (learn.longtimenohack.com .../quantization.html,
// the Blackwell FP4 paragraph): block-scaled FP4 goes straight to the tensor
// cores instead of being dequantized to 16-bit first.  The page's own sketch
// unpacks FP4 to FP8 in registers before an FP8 product; on B200 the tensor
// core reads FP4 and FP8 operands and both scale vectors itself, so no
// per-element instruction remains between HBM and the MMA.
//
// B200 design.  The MMA computes the transposed tile
//     D[128 weight rows, BN tokens] += (W^ . X^^T) over 32 k per instruction
// with both operands K-major in shared memory (128-byte swizzle):
//   * A = the FP4 weight codes.  kind::mxf8f6f4 takes 4-bit operands in
//     shared memory with each 16-element (8-byte) chunk followed by an 8-byte
//     gap; TMA writes that form itself (the 16U4_ALIGN16B tensor type), so
//     the packed codes travel from HBM at 4 bits per weight and nothing
//     touches them on the way;
//   * B = the E4M3 activation codes, a [BN tokens x 128 k] byte box;
//   * the E8M0 scales of both operands are stored in the tensor-core layout
//     (w4_mx_scale_layout, w4_mxfp8_quant): one 512-byte atom per 128 rows x
//     128 k, fetched with one bulk copy per stage and moved to tensor memory
//     with tcgen05.cp (32 lanes x 128 bits, broadcast to the four lane
//     quarters); the MMA of k-step kb reads byte kb of each 32-bit column;
//   * D lives in tensor memory (BN fp32 columns) and is read back with
//     tcgen05.ld, one weight row per lane, so a warp writes 32 consecutive
//     outputs of one token.
// Warp roles (192 threads): warp 0 issues the copies, warp 1 allocates tensor
// memory and one of its threads issues tcgen05.cp and the MMAs, warps 2..5
// run the epilogue.  A ring of stages couples producer and issuer with
// mbarriers (full: the stage's bytes landed; empty: tcgen05.commit after the
// MMAs that read it).  The scale columns alternate between two slots so that
// the copy for one stage never overwrites scales an MMA may still read.
//
// Split-K: when the tile grid leaves SMs idle, the 128-wide k-stages are split
// across the CTAs of a thread-block cluster (at most 8), sized so that every
// CTA of the grid is resident at once.  Each CTA parks its fp32 partial tile in
// its own (by then idle) shared memory; after a cluster barrier the first CTA
// of the cluster reads the others' partials through distributed shared memory,
// sums them in split order (the result does not depend on timing) and writes
// Y; a second cluster barrier keeps every partial alive until it has been read.
// With W4_WEIGHTS_STATIC the weight copies of the first ring of stages are
// issued before the kernel waits for the previous one on the stream; the
// activations wait.  (An L2 prefetch of the rest of each CTA's weight slice at
// that point made the kernel slower and is not done.)
// Every wait on a copy or an MMA is bounded in time; a wait that runs out
// records an error code (read by w4_device_error), raises a CTA-wide abort
// flag, and the CTA drains its own copies and MMAs, takes part in the cluster
// barriers, frees its tensor memory and returns.
#include "common.cuh"
#include "tc_ptx.cuh"

#include <cuda.h>

namespace w4 {
namespace {

constexpr int kMxThreads = 192;
constexpr int kMxKS = 128;                      // k per stage (four MMA k-steps of 32)

enum : int { kErrMxWaitEmpty = 0x301, kErrMxWaitFull = 0x302, kErrMxWaitDone = 0x303, kErrMxDrain = 0x304 };

template <int BN>
struct MxCfg {
    static constexpr int kSfb = (BN + 127) / 128;           // scale atoms of the activation tile
    static constexpr int kABytes = 128 * 128;                // 128 rows x 128 k, one byte per element in smem
    static constexpr int kBBytes = BN * 128;
    static constexpr int kSfaOff = kABytes + kBBytes;
    static constexpr int kSfbOff = kSfaOff + 512;
    static constexpr int kStageBytes = (kSfbOff + 512 * kSfb + 1023) / 1024 * 1024;
    static constexpr int kPerSM = BN <= 64 ? 2 : 1;          // CTAs per SM
    static constexpr int kBudget = (kPerSM == 2 ? 113 : 226) * 1024 - 1024 - 256;
    static constexpr int kStages = kBudget / kStageBytes > 8 ? 8 : kBudget / kStageBytes;
    static constexpr int kSmem = 1024 + kStages * kStageBytes + 256;
    static constexpr int kSfCols = 4 * (1 + kSfb);           // one slot: SFA (4 columns) then SFB
    static constexpr int kUsedCols = BN + 2 * kSfCols;
    static constexpr int kCols = kUsedCols <= 32 ? 32 : kUsedCols <= 64 ? 64 : kUsedCols <= 128 ? 128
                               : kUsedCols <= 256 ? 256 : 512;
    // kind::mxf8f6f4 block-scaled descriptor: A = E2M1 (5), B = E4M3 (0), both
    // K-major, N = BN, E8M0 scales (bit 23), M = 128; the scale byte ids
    // (bits 4-5 for B, 29-30 for A) are OR-ed in per k-step
    static constexpr uint32_t kIdesc = (5u << 7) | (0u << 10) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) |
                                       ((uint32_t)(128 >> 4) << 24);
    static_assert(kStages >= 2, "shared memory too small for the ring");
    static_assert(kStageBytes % 1024 == 0 && kABytes % 1024 == 0 && kBBytes % 1024 == 0, "swizzle atom alignment");
    static_assert(kUsedCols <= 512, "tensor memory overflow");
};

__device__ __forceinline__ void bulk_load(void *dst, const void *src, uint32_t bytes, uint64_t *bar)
{
    asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];" ::"r"(
                     smem_u32(dst)),
                 "l"(src), "r"(bytes), "r"(smem_u32(bar))
                 : "memory");
}

// 32 rows x 16 bytes of shared memory -> tensor memory lanes 0..31 of four
// 32-bit columns, repeated in all four lane quarters.
__device__ __forceinline__ void tmem_cp_sf(uint32_t taddr, uint64_t sdesc)
{
    asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}

// Shared-memory descriptor of a 512-byte scale atom (32 rows of 16 bytes, no
// swizzle): 8-row core matrices 128 bytes apart (stride byte offset), one core
// matrix along k, descriptor version 1.
__device__ __forceinline__ uint64_t desc_sf_atom(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

__device__ __forceinline__ void mma_mx(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %6, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%4], [%5], p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
        : "memory");
}

__device__ __forceinline__ void cluster_sync_all()
{
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

__device__ __forceinline__ uint32_t cluster_rank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// The shared::cluster address of `addr` (a shared::cta address) in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_cluster(uint32_t addr, uint32_t rank)
{
    uint32_t r;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
    return r;
}

__device__ __forceinline__ float ld_cluster_f32(uint32_t addr)
{
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
    return v;
}

__device__ __noinline__ bool mx_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, int *err, int code,
                                     uint64_t limit)
{
    if (mbar_try_wait(bar, parity)) return true;
    const uint64_t t0 = globaltimer();
    while (true) {
        if (mbar_try_wait(bar, parity)) return true;
        if (*abort_flag) return false;
        if (globaltimer() - t0 > limit) {
            *abort_flag = 1;
            atomicCAS(err, 0, code);
            return false;
        }
    }
}

// Ignores the abort flag; bounded by the default limit only.
__device__ __noinline__ void mx_drain(uint64_t *bar, uint32_t parity, int *err)
{
    const uint64_t t0 = globaltimer();
    while (!mbar_try_wait(bar, parity)) {
        if (globaltimer() - t0 > kDefaultWaitNs) {
            atomicCAS(err, 0, kErrMxDrain);
            return;
        }
    }
}

template <int BN, bool EARLY>
__global__ void __launch_bounds__(kMxThreads, MxCfg<BN>::kPerSM)
mx_gemm_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
               const uint8_t *__restrict__ w_sf, const uint8_t *__restrict__ x_sf, int M, int N, int K,
               __nv_bfloat16 *__restrict__ Y, int splits, int ks_per_split, int *err, uint64_t wait_ns)
{
    using C = MxCfg<BN>;
    constexpr int S = C::kStages;
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
    uint64_t *full = (uint64_t *)(smem + S * C::kStageBytes);
    uint64_t *empty = full + S;
    uint64_t *done = empty + S;
    uint64_t *stall = done + 1;                       // a barrier nothing completes (failure tests)
    uint32_t *tmem_slot = (uint32_t *)(stall + 1);
    volatile int *abort_flag = (volatile int *)(tmem_slot + 1);
    const uint64_t limit = wait_limit_of(wait_ns);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int n0 = blockIdx.x * 128, m0 = blockIdx.y * BN, split = blockIdx.z;
    const int KS = K / kMxKS;
    const int ks_begin = split * ks_per_split;
    const int nks = min(KS, ks_begin + ks_per_split) - ks_begin;
    // activation scale atoms this tile reads (the last 128-row band may hold
    // fewer than kSfb atoms), and the tensor-memory column shift of a tile
    // that starts inside an atom (BN < 128: m0 % 128 rows = (m0 % 128) / 32 columns)
    const int bands = (M + 127) >> 7;
    const int nsfb = min(C::kSfb, bands - (m0 >> 7));
    const uint32_t sfb_shift = (uint32_t)((m0 & 127) >> 5);

    if (threadIdx.x == 0) {
        for (int s = 0; s < S; ++s) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        mbar_init(done, 1);
        mbar_init(stall, 1);
        *abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1) tmem_alloc(tmem_slot, C::kCols);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    const uint32_t tx = 128 * kMxKS / 2 + C::kBBytes + 512 + 512 * nsfb;
    const uint8_t *sfa_src = w_sf + ((size_t)(n0 >> 7) * KS + ks_begin) * 512;
    const uint8_t *sfb_src = x_sf + ((size_t)(m0 >> 7) * KS + ks_begin) * 512;
    const int first = min(nks, S);               // stages whose ring slots are free at the start
    auto issue_w = [&](int i) {                  // weight half of stage i (codes + scale atom)
        const int s = i % S;
        uint8_t *st = smem + s * C::kStageBytes;
        tma_load_2d(st, &tmap_w, &full[s], (ks_begin + i) * kMxKS, n0);
        bulk_load(st + C::kSfaOff, sfa_src + (size_t)i * 512, 512, &full[s]);
    };
    auto issue_x = [&](int i) {                  // activation half of stage i
        const int s = i % S;
        uint8_t *st = smem + s * C::kStageBytes;
        tma_load_2d(st + C::kABytes, &tmap_x, &full[s], (ks_begin + i) * kMxKS, m0);
        for (int j = 0; j < nsfb; ++j)
            bulk_load(st + C::kSfbOff + 512 * j, sfb_src + ((size_t)j * KS + i) * 512, 512, &full[s]);
    };
    if (EARLY && warp == 0 && lane == 0) {
        // the weights are not written by the previous kernel: start streaming them now
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_w) : "memory");
        for (int i = 0; i < first; ++i) {
            mbar_arrive_expect_tx(&full[i], tx);
            issue_w(i);
        }
    }
    pdl_wait();                                   // the activations (and, without EARLY, everything) are ready
    pdl_launch_dependents();

    if (warp == 0) {
        // ------------------------------------------------ copy producer --
        if (lane == 0) {
            if (!EARLY) asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_w) : "memory");
            asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_x) : "memory");
            int issued = 0;
            if (EARLY) {
                for (int i = 0; i < first; ++i) issue_x(i);
                issued = first;
            }
            for (int i = issued; i < nks; ++i) {
                const int s = i % S;
                const uint32_t ph = (i / S) & 1;
                if (!mx_wait(&empty[s], ph ^ 1, abort_flag, err, kErrMxWaitEmpty, limit)) break;
                mbar_arrive_expect_tx(&full[s], tx);
                issue_w(i);
                issue_x(i);
                ++issued;
            }
            // every issued copy must have landed before the CTA may exit
            for (int i = max(0, issued - S); i < issued; ++i) mx_drain(&full[i % S], (i / S) & 1, err);
        }
    } else if (warp == 1) {
        // ------------------------------------------------- MMA issuer ---
        if (lane == 0) {
            const uint64_t desc0 = desc_k_sw128(smem_u32(smem));
            const uint32_t sf0 = smem_u32(smem) + C::kSfaOff;
            for (int i = 0; i < nks; ++i) {
                const int s = i % S;
                const uint32_t ph = (i / S) & 1;
                // (the issuer's first wait targets a barrier that nothing
                // completes in the failure-path tests)
                uint64_t *fb = (i == 0 && stalls_first_wait(wait_ns)) ? stall : &full[s];
                if (!mx_wait(fb, fb == stall ? 0u : ph, abort_flag, err, kErrMxWaitFull, limit)) break;
                tc_fence_after();
                const uint32_t slot = tmem + BN + (uint32_t)((i & 1) * C::kSfCols);
                const uint32_t sfa_t = slot, sfb_t = slot + 4;
                const uint32_t soff = (uint32_t)(s * C::kStageBytes);
                tmem_cp_sf(sfa_t, desc_sf_atom(sf0 + soff));
                for (int j = 0; j < nsfb; ++j) tmem_cp_sf(sfb_t + 4 * j, desc_sf_atom(sf0 + soff + 512 + 512 * j));
                const uint64_t ad = desc0 + (soff >> 4), bd = desc0 + ((soff + C::kABytes) >> 4);
#pragma unroll
                for (int kb = 0; kb < 4; ++kb) {
                    const uint32_t id = C::kIdesc | ((uint32_t)kb << 4) | ((uint32_t)kb << 29);
                    mma_mx(tmem, ad + 2 * kb, bd + 2 * kb, id, sfa_t | ((uint32_t)kb << 30),
                           (sfb_t + sfb_shift) | ((uint32_t)kb << 30), (i | kb) != 0 ? 1u : 0u);
                }
                mma_commit(&empty[s]);
            }
            mma_commit(done);
            mx_drain(done, 0, err);   // no MMA or copy may still run when tensor memory is freed
        }
        __syncwarp();
    } else {
        // --------------------------------------------------- epilogue ---
        const int q = warp & 3;                      // tensor-memory lane quarter of this warp
        const int n = n0 + 32 * q + lane;
        const bool okn = n < N;
        const uint32_t lane_addr = tmem + ((uint32_t)(32 * q) << 16);
        const bool have =
            __all_sync(0xffffffffu, mx_wait(done, 0, abort_flag, err, kErrMxWaitDone, limit) && *abort_flag == 0);
        tc_fence_after();
        // columns (tokens) of this tile that exist
        const int cols = min(BN, M - m0);
        float *red = (float *)smem;                  // [BN][128] fp32 partial, in the idle ring
        if (have) {
            constexpr int CH = BN < 32 ? BN : 32;
            for (int c = 0; c < cols; c += CH) {
                float acc[CH];
                if constexpr (CH == 32) {
                    tmem_ld32(lane_addr + c, acc);
                } else {
#pragma unroll
                    for (int u = 0; u < CH / 8; ++u) tmem_ld8(lane_addr + c + 8 * u, acc + 8 * u);
                }
                tmem_wait_ld();
#pragma unroll
                for (int j = 0; j < CH; ++j) {
                    if (c + j < cols) {
                        if (splits == 1) {
                            if (okn) Y[(size_t)(m0 + c + j) * N + n] = __float2bfloat16_rn(acc[j]);
                        } else {
                            red[(c + j) * 128 + 32 * q + lane] = acc[j];
                        }
                    }
                }
            }
        }
    }

    if (splits > 1) {
        // split-K across the cluster: partials are summed in split order by the
        // cluster's first CTA (every thread of every CTA takes part in both
        // barriers, also after an abort, when Y is left undefined)
        cluster_sync_all();
        if (cluster_rank() == 0 && warp >= 2) {
            const int q = warp & 3;
            const int r = 32 * q + lane;
            const int n = n0 + r;
            const int cols = min(BN, M - m0);
            const uint32_t red0 = smem_u32(smem);
            if (n < N) {
                for (int c = 0; c < cols; ++c) {
                    const uint32_t a = red0 + (uint32_t)((c * 128 + r) * 4);
                    float v[8];
#pragma unroll
                    for (int sp = 0; sp < 8; ++sp)
                        if (sp < splits) v[sp] = ld_cluster_f32(map_cluster(a, (uint32_t)sp));
                    float sum = v[0];
#pragma unroll
                    for (int sp = 1; sp < 8; ++sp)
                        if (sp < splits) sum += v[sp];
                    Y[(size_t)(m0 + c) * N + n] = __float2bfloat16_rn(sum);
                }
            }
        }
        cluster_sync_all();
    }

    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    if (warp == 1) tmem_dealloc(tmem, C::kCols);
}

// ----------------------------------------------------------------- host --

struct MxPlan {
    int BN = 0, m_tiles = 0, n_tiles = 0, splits = 1, ks_per_split = 0;
};

constexpr int kMxMaxSplits = 8;                 // portable cluster size

int mx_pick_bn(int64_t M)
{
    if (M <= 16) return 16;
    if (M <= 32) return 32;
    if (M <= 64) return 64;
    if (M <= 128) return 128;
    return 256;
}

MxPlan plan_mx(int64_t M, int64_t N, int64_t K)
{
    MxPlan p;
    p.BN = mx_pick_bn(M);
    p.m_tiles = (int)((M + p.BN - 1) / p.BN);
    p.n_tiles = (int)((N + 127) / 128);
    const int KS = (int)(K / kMxKS);
    const int64_t tiles = (int64_t)p.m_tiles * p.n_tiles;
    const int64_t slots = (int64_t)kNumSMs * (p.BN <= 64 ? 2 : 1);
    // the most splits (at least two k-stages each, at most one cluster) whose
    // grid is resident at once: HBM is then shared by every CTA of the grid and
    // none waits for a second wave.  Clusters are placed within GPCs, which
    // strands some CTA slots: a grid of 96 three-CTA clusters (288 CTAs of 296
    // slots) ran partly in a second wave, 86 of them (258 CTAs) did not, so
    // split grids keep 10% of the slots free.
    const int64_t cluster_slots = slots * 9 / 10;
    int per = KS;
    for (int s = 2; s <= KS / 2 && s <= kMxMaxSplits; ++s) {
        const int per_s = (KS + s - 1) / s;
        const int s_eff = (KS + per_s - 1) / per_s;
        if (tiles * s_eff > cluster_slots) break;
        per = per_s;
    }
    p.ks_per_split = per;
    p.splits = (KS + per - 1) / per;
    return p;
}

template <int BN, bool EARLY>
cudaError_t mx_launch_bn(const CUtensorMap &wmap, const CUtensorMap &xmap, const MxPlan &p, int M, int N, int K,
                         const uint8_t *w_codes, const uint8_t *w_sf, const uint8_t *x_sf, void *Y,
                         cudaStream_t stream)
{
    using C = MxCfg<BN>;
    auto kern = mx_gemm_kernel<BN, EARLY>;
    static std::atomic<bool> attr_done[kMaxDevices];
    {
        const cudaError_t e = set_smem_attr(kern, C::kSmem, attr_done);
        if (e != cudaSuccess) return e;
    }
    int *err = device_error_word();
    if (!err) return cudaErrorUnknown;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(p.n_tiles, p.m_tiles, p.splits);
    cfg.blockDim = dim3(kMxThreads);
    cfg.dynamicSmemBytes = C::kSmem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = 1;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = (unsigned)p.splits;
    cfg.attrs = attr;
    cfg.numAttrs = p.splits > 1 ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, kern, wmap, xmap, w_sf, x_sf, M, N, K, (__nv_bfloat16 *)Y, p.splits,
                              p.ks_per_split, err, wait_limit_ns());
}

template <int BN>
cudaError_t mx_launch_early(bool early, const CUtensorMap &wmap, const CUtensorMap &xmap, const MxPlan &p, int M,
                            int N, int K, const uint8_t *w_codes, const uint8_t *w_sf, const uint8_t *x_sf, void *Y,
                            cudaStream_t stream)
{
    if (early) return mx_launch_bn<BN, true>(wmap, xmap, p, M, N, K, w_codes, w_sf, x_sf, Y, stream);
    return mx_launch_bn<BN, false>(wmap, xmap, p, M, N, K, w_codes, w_sf, x_sf, Y, stream);
}

}  // namespace

cudaError_t launch_mx_gemm(const uint8_t *x_codes, const uint8_t *x_sf, int64_t M, int64_t N, int64_t K,
                           const uint8_t *w_codes, const uint8_t *w_sf, void *Y, bool weights_static,
                           cudaStream_t stream)
{
    const MxPlan p = plan_mx(M, N, K);
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    const cuuint32_t estride[2] = {1, 1};
    // weights: 4-bit codes [N][K], unpacked by TMA into 16-byte chunks of 16
    // codes + 8 bytes of gap (the operand form of kind::mxf8f6f4)
    CUtensorMap wmap;
    const cuuint64_t wdim[2] = {(cuuint64_t)K, (cuuint64_t)N};
    const cuuint64_t wstride[1] = {(cuuint64_t)K / 2};
    const cuuint32_t wbox[2] = {(cuuint32_t)kMxKS, 128u};
    if (enc(&wmap, CU_TENSOR_MAP_DATA_TYPE_16U4_ALIGN16B, 2, const_cast<uint8_t *>(w_codes), wdim, wstride, wbox,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    // activations: E4M3 bytes [M][K]
    CUtensorMap xmap;
    const cuuint64_t xdim[2] = {(cuuint64_t)K, (cuuint64_t)M};
    const cuuint64_t xstride[1] = {(cuuint64_t)K};
    const cuuint32_t xbox[2] = {(cuuint32_t)kMxKS, (cuuint32_t)p.BN};
    if (enc(&xmap, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t *>(x_codes), xdim, xstride, xbox, estride,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return cudaErrorInvalidValue;
    const bool e = weights_static;
    switch (p.BN) {
    case 16: return mx_launch_early<16>(e, wmap, xmap, p, (int)M, (int)N, (int)K, w_codes, w_sf, x_sf, Y, stream);
    case 32: return mx_launch_early<32>(e, wmap, xmap, p, (int)M, (int)N, (int)K, w_codes, w_sf, x_sf, Y, stream);
    case 64: return mx_launch_early<64>(e, wmap, xmap, p, (int)M, (int)N, (int)K, w_codes, w_sf, x_sf, Y, stream);
    case 128: return mx_launch_early<128>(e, wmap, xmap, p, (int)M, (int)N, (int)K, w_codes, w_sf, x_sf, Y, stream);
    default: return mx_launch_early<256>(e, wmap, xmap, p, (int)M, (int)N, (int)K, w_codes, w_sf, x_sf, Y, stream);
    }
}

}  // namespace w4
