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
// Budget.  At the measured HBM bandwidth the 148 SMs can issue about 2.9
// thread instructions per weight (0.52 B per weight at g = 128), and the
// exact dequantization alone takes 19 instructions per packed word of 8
// weights (2.4 per weight).  So the kernel is as much issue-bound as
// HBM-bound, and everything besides the dequantization has to cost next to
// nothing:
//   * a CTA (4 warps, 8 when there are few tiles) owns a tile of 16 output
//     channels and all of K; warp w takes the SK-wide k-stages w, w+NW, ...
//     and the partial tiles are summed in shared memory at the end (no
//     global scratch); the launch keeps every CTA resident in one wave;
//   * the codes stream HBM -> shared memory by TMA, one 2-D box of 16 rows x
//     128 bytes (256 k) with the 128-byte swizzle per box, SK/256 boxes per
//     stage, R stages in flight per warp on the warp's own mbarrier ring;
//   * per stage, each lane turns 16 * SK / G / 32 (channel, group) scales and
//     zero-points into the bf16x2 constants below and parks them in the
//     warp's shared-memory slot, where the lanes that need them read them
//     back (the next stage's scales and zero-points are loaded during this
//     one, and the tile's whole rows are asked into L2 at launch);
//   * lane (g, t) = (lane/4, lane%4) reads, for channels g and g+8, the 16-byte
//     chunks t and t+4 of each box (the swizzle makes these reads free of bank
//     conflicts); every shared-memory offset is a per-lane constant plus a
//     compile-time one;
//   * the activations of a chunk come from global memory (they stay in L1:
//     every CTA of the SM reads the same few KB);
//   * when the caller declares the packed weight static (W4_WEIGHTS_STATIC:
//     the kernel before this one on the stream does not write it), the code
//     copies, and the scale and zero-point loads, start before the
//     programmatic dependency on that kernel resolves, so in a decode loop
//     the weight stream of one layer overlaps the tail of the previous
//     kernel; only the activations wait for it;
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
#include "tc_ptx.cuh"

namespace w4 {
namespace {

constexpr int kErrGemvWait = 0x201, kErrGemvDrain = 0x202;

// Bounded wait for the phase with the given parity of the barrier at shared
// address `bar`; false after `limit` ns (a box lands in microseconds).
__device__ __noinline__ bool gemv_wait(uint32_t bar, uint32_t parity, uint64_t limit = kDefaultWaitNs)
{
    auto test = [&]() {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        return ok != 0;
    };
    if (test()) return true;
    const uint64_t t0 = globaltimer();
    while (!test())
        if (globaltimer() - t0 > limit) return false;
    return true;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1)
{
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
        "{%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// Kernel shape: SK k per stage (SK/256 code boxes), R stages in flight per
// warp, NW warps per CTA.
template <int G, int SK, int NW, int R, int MT>
struct GemvCfg {
    static constexpr int kBoxes = SK / 256;
    static constexpr int kBoxBytes = 16 * 128;
    static constexpr int kStageBytes = kBoxes * kBoxBytes;
    static constexpr int kGroups = SK / G;            // groups per stage and channel
    static constexpr int kConsts = 16 * kGroups;      // constants per warp and stage
    static constexpr int kCpl = kConsts / 32;         // computed per lane and stage
    static constexpr int kChunks = 2 * kBoxes;        // 32-k chunks per lane and stage
    static constexpr int kConstOff = NW * R * kStageBytes;
    static constexpr int kBarOff = kConstOff + NW * kConsts * 16;
    static constexpr int kStallOff = kBarOff + NW * R * 8;      // a barrier nothing completes (failure tests)
    static constexpr int kBytes = kStallOff + 8 + 1024;          // + alignment slack
    static_assert(SK % 256 == 0 && kCpl >= 1, "stage shape");
    static_assert(32 * 4 * MT * 4 <= R * kStageBytes, "the reduction reuses each warp's stage ring");
};

// bf16x2 constants of one (channel, group): s_hi, s_lo and -(128 + zp), each
// duplicated into both halves (w^ = 0 for s16 = 0).
__device__ __forceinline__ uint4 const_word(unsigned short s16bits, uint32_t zp)
{
    const GroupConst c = group_const(s16bits, zp);
    return make_uint4(c.shi, c.slo, c.z, 0u);
}

template <int G, int MODE, int MT, int NW, int SK, int R, int MINB, bool EARLY, bool XPF>
__global__ void __launch_bounds__(NW * 32, MINB)
gemv_kernel(const __grid_constant__ CUtensorMap tmap_q, const __nv_bfloat16 *__restrict__ X, int M, int N, int K,
            const unsigned short *__restrict__ scales, const uint32_t *__restrict__ qzeros,
            void *__restrict__ Y, int yflags, int *err, uint64_t wait_ns)
{
    // bit 0: fp32 Y (W4_OUT_F32); bit 1: codes in the repacked layout
    // (w4_repack: 2 KB boxes stored contiguously, the tensor map is 4-D)
    const int y_f32 = yflags & 1;
    const bool repacked = (yflags & 2) != 0;
    using C = GemvCfg<G, SK, NW, R, MT>;
    extern __shared__ uint8_t smem_raw[];
    // (an offset from the shared array, not an integer cast, so that the
    // compiler keeps the shared address space and emits shared loads)
    uint8_t *smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);

    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    const int g = lane >> 2, t = lane & 3;
    const int NG = K / G, ZW = (NG + 7) >> 3;
    const int NS = (K + SK - 1) / SK;                 // stages per channel
    const int nsw = NS > warp ? (NS - warp + NW - 1) / NW : 0;   // stages of this warp
    const int r0 = (int)blockIdx.x * 16;

    uint8_t *ring = smem + warp * R * C::kStageBytes;
    uint4 *cslot = (uint4 *)(smem + C::kConstOff) + warp * C::kConsts;
    const uint32_t ring_s = smem_u32(ring);
    const uint32_t bar0 = smem_u32(smem + C::kBarOff) + warp * R * 8;
    const uint32_t stall_bar = smem_u32(smem + C::kStallOff);
    const uint64_t limit = wait_limit_of(wait_ns);

    if (lane == 0) {
        for (int s = 0; s < R; ++s) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8 * s));
        if (warp == 0) asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(stall_bar));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_q) : "memory");
    }
    __syncthreads();
    // With EARLY (the caller declared that the kernel before this one on the
    // stream does not write the packed weight), the weight stream starts
    // before the programmatic dependency resolves, overlapping that kernel's
    // tail; only the activations wait.  Otherwise everything waits.
    if (!EARLY) {
        pdl_wait();                                   // the previous kernel's writes are visible
        pdl_launch_dependents();
    }

    auto issue = [&](int i) {                         // lane 0: stage i of this warp into slot i % R
        const int s = i % R;
        const int sb = warp + NW * i;
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar0 + 8 * s),
                     "r"(C::kStageBytes)
                     : "memory");
#pragma unroll
        for (int bb = 0; bb < C::kBoxes; ++bb) {      // a box past the end of K is zero-filled
            if (repacked)
                asm volatile(
                    "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %3, "
                    "%4, %5}], [%2];" ::"r"(ring_s + s * C::kStageBytes + bb * C::kBoxBytes),
                    "l"(&tmap_q), "r"(bar0 + 8 * s), "r"(0), "r"(sb * C::kBoxes + bb), "r"(r0 >> 4)
                    : "memory");
            else
                asm volatile(
                    "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, "
                    "%4}], [%2];" ::"r"(ring_s + s * C::kStageBytes + bb * C::kBoxBytes),
                    "l"(&tmap_q), "r"(bar0 + 8 * s), "r"((sb * C::kBoxes + bb) * 32), "r"(r0)
                    : "memory");
        }
    };
    if (lane == 0)
        for (int i = 0; i < R && i < nsw; ++i) issue(i);
    if (threadIdx.x == 32) {                          // the tile's scales and zero-points, HBM -> L2
        const int rows = min(16, N - r0);
        prefetch_l2(scales + (size_t)r0 * NG, (size_t)rows * NG * 2);
        if (MODE == W4_ASYM) prefetch_l2(qzeros + (size_t)r0 * ZW, (size_t)rows * ZW * 4);
    }

    // scales / zero-points of the constants this lane computes for stage i
    unsigned short sv[C::kCpl];
    uint32_t zv[C::kCpl];
    auto load_consts = [&](int i) {
        const int sb = warp + NW * i;
#pragma unroll
        for (int u = 0; u < C::kCpl; ++u) {
            const int idx = lane + 32 * u, row = r0 + (idx & 15), j = sb * C::kGroups + (idx >> 4);
            const bool ok = row < N && j < NG;
            sv[u] = ok ? __ldg(scales + (size_t)row * NG + j) : (unsigned short)0;
            if (MODE == W4_ASYM) zv[u] = ok ? (__ldg(qzeros + (size_t)row * ZW + (j >> 3)) >> (4 * (j & 7))) & 0xFu : 0u;
            else zv[u] = 8u;
        }
    };
    if (nsw > 0) load_consts(0);
    if (EARLY) {
        pdl_wait();                                   // the activations come from the previous kernel
        pdl_launch_dependents();
    }

    // per-lane constant parts of the shared-memory offsets
    const int offA = g * 128 + ((t ^ g) << 4);        // chunk t of row g (chunk t + 4: offA ^ 64)
    const int lane_gl = G == 128 ? 0 : G == 64 ? (t >> 1) : t;
    const uint4 *clane = cslot + g + 16 * lane_gl;    // constants of row g (row g + 8: + 8)
    const __nv_bfloat16 *xrow[MT];                   // a token past M reads token M-1
#pragma unroll
    for (int mt = 0; mt < MT; ++mt) xrow[mt] = X + (size_t)min(g + 8 * mt, M - 1) * K + t * 32;

    // activations of chunk h of stage sb: 4 x 16 bytes per token group.  In a
    // stage that runs past the end of K (K is a multiple of 32, chunks are
    // whole) a chunk past the end reads the last chunk's activations instead:
    // its codes are zero-filled by TMA and its groups' constants have
    // s16 = 0, so every w^ there is 0 and the activations only need to be finite
    auto load_x = [&](uint4 (&xv)[MT][4], int sb, int h) {
        const int kc = sb * SK + (h >> 1) * 256 + (h & 1) * 128;   // this lane adds t * 32
        const int kk = (sb + 1) * SK <= K ? kc : min(kc + t * 32, K - 32) - t * 32;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt)
#pragma unroll
            for (int w = 0; w < 4; ++w) xv[mt][w] = __ldg((const uint4 *)(xrow[mt] + kk) + w);
    };

    // two accumulator sets (the first and the second MMA of every word pair)
    // halve the dependent chain of MMAs
    float acc[MT][4], acc2[MT][4];
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) acc[mt][e] = acc2[mt][e] = 0.f;

    uint4 xn[MT][4];
    if (XPF && nsw > 0) load_x(xn, warp, 0);
    const uint32_t magic = 0x43004300u;              // bf16x2 of (128, 128)

    bool ok = true;
    int i = 0;
    for (; i < nsw; ++i) {
        const int sb = warp + NW * i;
        const int s = i % R;
        // constants of this stage into the warp's slot, then the next stage's loads
        __syncwarp();                                 // every lane is done with the previous stage's slot
#pragma unroll
        for (int u = 0; u < C::kCpl; ++u) cslot[lane + 32 * u] = const_word(sv[u], zv[u]);
        if (i + 1 < nsw) load_consts(i + 1);
        __syncwarp();
        const bool stall = i == 0 && stalls_first_wait(wait_ns);   // failure-path tests only
        if (!gemv_wait(stall ? stall_bar : bar0 + 8 * s, stall ? 0u : (uint32_t)(i / R) & 1u, limit)) {
            ok = false;
            break;
        }
        const uint8_t *st = ring + s * C::kStageBytes;
#pragma unroll
        for (int h = 0; h < C::kChunks; ++h) {
            const int bb = h >> 1, odd = h & 1;
            uint4 xc[MT][4];
            if (XPF) {
#pragma unroll
                for (int mt = 0; mt < MT; ++mt)
#pragma unroll
                    for (int w = 0; w < 4; ++w) xc[mt][w] = xn[mt][w];
                if (h + 1 < C::kChunks) load_x(xn, sb, h + 1);
                else if (i + 1 < nsw) load_x(xn, sb + NW, 0);
            } else {
                load_x(xc, sb, h);
            }
            // this lane's codes: channels g and g+8, chunk t + 4 * odd (128-byte swizzle)
            const uint8_t *cp = st + bb * C::kBoxBytes + (offA ^ (odd * 64));
            const uint4 wa4 = *(const uint4 *)cp;
            const uint4 wb4 = *(const uint4 *)(cp + 8 * 128);
            const int coff = 16 * ((bb * 256 + odd * 128) / G);
            const uint4 ca4 = clane[coff], cb4 = clane[coff + 8];
            const GroupConst ca = {ca4.x, ca4.y, ca4.z}, cb = {cb4.x, cb4.y, cb4.z};
            const uint32_t wa[4] = {wa4.x, wa4.y, wa4.z, wa4.w};
            const uint32_t wb[4] = {wb4.x, wb4.y, wb4.z, wb4.w};
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                const uint32_t a0 = dequant_pair(wa[w], 0, ca, magic), a1 = dequant_pair(wa[w], 1, ca, magic);
                const uint32_t a2 = dequant_pair(wa[w], 2, ca, magic), a3 = dequant_pair(wa[w], 3, ca, magic);
                const uint32_t b0 = dequant_pair(wb[w], 0, cb, magic), b1 = dequant_pair(wb[w], 1, cb, magic);
                const uint32_t b2 = dequant_pair(wb[w], 2, cb, magic), b3 = dequant_pair(wb[w], 3, cb, magic);
#pragma unroll
                for (int mt = 0; mt < MT; ++mt) {
                    mma_bf16_16816(acc[mt], a0, b0, a1, b1, xc[mt][w].x, xc[mt][w].y);
                    mma_bf16_16816(acc2[mt], a2, b2, a3, b3, xc[mt][w].z, xc[mt][w].w);
                }
            }
        }
        __syncwarp();                                 // the stage is read: refill it
        if (lane == 0 && i + R < nsw) {
            asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
            issue(i + R);
        }
    }
    if (!ok) {
        // a box never landed: record it, wait (bounded) for the copies this warp
        // still has in flight, and leave the tile unwritten
        if (lane == 0) {
            atomicCAS(err, 0, kErrGemvWait);
            for (int j = i; j < nsw && j < i + R; ++j)
                if (!gemv_wait(bar0 + 8 * (j % R), (uint32_t)(j / R) & 1u)) atomicCAS(err, 0, kErrGemvDrain);
        }
    }

    // cross-warp reduction: each warp parks its partial tile in its own (now
    // idle) stage ring, whose copies have all landed
    __syncwarp();
    float(*myred)[4 * MT] = (float(*)[4 * MT])ring;
#pragma unroll
    for (int mt = 0; mt < MT; ++mt)
#pragma unroll
        for (int e = 0; e < 4; ++e) myred[lane][4 * mt + e] = acc[mt][e] + acc2[mt][e];
    const int all_ok = __syncthreads_and(ok ? 1 : 0);
    if (warp == 0 && all_ok) {
        const int rA = r0 + g, rB = rA + 8;
#pragma unroll
        for (int mt = 0; mt < MT; ++mt) {
            float sm[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
            for (int w = 0; w < NW; ++w)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    sm[e] += ((const float(*)[4 * MT])(smem + w * R * C::kStageBytes))[lane][4 * mt + e];
            const int m0 = 8 * mt + 2 * t, m1 = m0 + 1;   // tokens of c0/c2 and c1/c3
            if (rA < N && m0 < M) store_y(Y, (size_t)m0 * N + rA, sm[0], y_f32);
            if (rA < N && m1 < M) store_y(Y, (size_t)m1 * N + rA, sm[1], y_f32);
            if (rB < N && m0 < M) store_y(Y, (size_t)m0 * N + rB, sm[2], y_f32);
            if (rB < N && m1 < M) store_y(Y, (size_t)m1 * N + rB, sm[3], y_f32);
        }
    }
}

template <int G, int MODE, int MT, int NW, int SK, int R, int MINB, bool EARLY = false, bool XPF = false>
cudaError_t launch_cfg(const CUtensorMap &map, const void *X, int64_t M, int64_t N, int64_t K, const void *scales,
                       const uint32_t *qzeros, void *Y, int y_f32, int *err, cudaStream_t stream)
{
    const int64_t blocks = (N + 15) / 16;             // one 16-channel tile per CTA
    constexpr int smem = GemvCfg<G, SK, NW, R, MT>::kBytes;
    static std::atomic<bool> attr_done[kMaxDevices];
    auto kern = gemv_kernel<G, MODE, MT, NW, SK, R, MINB, EARLY, XPF>;
    const cudaError_t e = set_smem_attr(kern, smem, attr_done);
    if (e != cudaSuccess) return e;
    return launch_pdl(kern, dim3((unsigned)blocks), dim3(NW * 32), smem, stream, map, (const __nv_bfloat16 *)X,
                      (int)M, (int)N, (int)K, (const unsigned short *)scales, qzeros, Y, y_f32, err,
                      wait_limit_ns());
}

// Launch shape by tile count (16 channels per tile), chosen from timings on
// the B200 so that every tile is resident in one wave where possible: at most
// two tiles per SM get 8 warps each (512-k stages); up to five per SM get 4
// warps (512-k stages); up to six per SM get 4 warps with 256-k stages, whose
// smaller ring and register budget let six CTAs share an SM.
template <int G, int MODE, int MT, bool EARLY>
cudaError_t launch_g(const CUtensorMap &map, const void *X, int64_t M, int64_t N, int64_t K, const void *scales,
                     const uint32_t *qzeros, void *Y, int y_f32, int *err, cudaStream_t stream)
{
    const int64_t tiles = (N + 15) / 16;
    if (tiles <= 2 * kNumSMs)
        return launch_cfg<G, MODE, MT, 8, 512, 2, 2, EARLY>(map, X, M, N, K, scales, qzeros, Y, y_f32, err, stream);
    if (MT == 1 && tiles > 5 * kNumSMs && tiles <= 6 * kNumSMs)
        return launch_cfg<G, MODE, MT, 4, 256, 2, 6, EARLY>(map, X, M, N, K, scales, qzeros, Y, y_f32, err, stream);
    return launch_cfg<G, MODE, MT, 4, 512, 2, (MT == 1 ? 5 : 4), EARLY>(map, X, M, N, K, scales, qzeros, Y, y_f32,
                                                                        err, stream);
}

template <int MT, bool EARLY>
cudaError_t launch_mt(const CUtensorMap &map, const void *X, int64_t M, int64_t N, int64_t K, const void *scales,
                      const uint32_t *qzeros, int group, int mode, void *Y, int y_f32, int *err,
                      cudaStream_t stream)
{
    switch (group * 2 + mode) {
    case 32 * 2 + W4_SYM: return launch_g<32, W4_SYM, MT, EARLY>(map, X, M, N, K, scales, qzeros, Y, y_f32, err, stream);
    case 32 * 2 + W4_ASYM: return launch_g<32, W4_ASYM, MT, EARLY>(map, X, M, N, K, scales, qzeros, Y, y_f32, err, stream);
    case 64 * 2 + W4_SYM: return launch_g<64, W4_SYM, MT, EARLY>(map, X, M, N, K, scales, qzeros, Y, y_f32, err, stream);
    case 64 * 2 + W4_ASYM: return launch_g<64, W4_ASYM, MT, EARLY>(map, X, M, N, K, scales, qzeros, Y, y_f32, err, stream);
    case 128 * 2 + W4_SYM: return launch_g<128, W4_SYM, MT, EARLY>(map, X, M, N, K, scales, qzeros, Y, y_f32, err, stream);
    case 128 * 2 + W4_ASYM: return launch_g<128, W4_ASYM, MT, EARLY>(map, X, M, N, K, scales, qzeros, Y, y_f32, err, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace

// The codes as a 2-D array of 32-bit words [N][K/8]; one box = 16 channels x
// 32 words (256 k) with the 128-byte swizzle.  Repacked codes (w4_repack) are
// the same boxes stored one after another: a 4-D array [ceil(N/16)][K/256][16]
// [32 words] whose box {32, 16, 1, 1} lands in shared memory exactly as the
// 2-D box does; a box at k-chunk K/256 or past it is out of range and
// zero-filled, as in the 2-D map.
cudaError_t gemv_code_map(CUtensorMap *map, const uint32_t *qweight, int64_t N, int64_t K, bool repacked)
{
    EncodeTiledFn enc = encode_fn();
    if (!enc) return cudaErrorNotSupported;
    CUresult cr;
    if (repacked) {
        const cuuint64_t gdim[4] = {32u, 16u, (cuuint64_t)(K / 256), (cuuint64_t)((N + 15) / 16)};
        const cuuint64_t gstride[3] = {128u, 2048u, (cuuint64_t)(K / 256) * 2048u};
        const cuuint32_t box[4] = {32u, 16u, 1u, 1u};
        const cuuint32_t estride[4] = {1u, 1u, 1u, 1u};
        cr = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 4, const_cast<uint32_t *>(qweight), gdim, gstride, box, estride,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    } else {
        const cuuint64_t gdim[2] = {(cuuint64_t)(K / 8), (cuuint64_t)N};
        const cuuint64_t gstride[1] = {(cuuint64_t)K / 2};
        const cuuint32_t box[2] = {32u, 16u};
        const cuuint32_t estride[2] = {1u, 1u};
        cr = enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 2, const_cast<uint32_t *>(qweight), gdim, gstride, box, estride,
                 CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                 CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    }
    return cr == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

// w4_repack: dst word (((n/16) * (K/256) + kw/32) * 16 + n%16) * 32 + kw%32 =
// qweight[n][kw] (0 for the rows that pad N to a multiple of 16); one thread
// per 4 words.
__global__ void __launch_bounds__(256) repack_kernel(const uint4 *__restrict__ q, int64_t N, int64_t K,
                                                     uint4 *__restrict__ out)
{
    pdl_wait();
    pdl_launch_dependents();
    const int64_t KW = K / 8, KC = K / 256;
    const int64_t total = (N + 15) / 16 * 16 * KW / 4;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (int64_t)gridDim.x * blockDim.x) {
        const int64_t w = i * 4;                           // first destination word
        const int64_t box = w / 512, in = w % 512;         // 16 rows x 32 words per box
        const int64_t t = box / KC, c = box % KC;
        const int64_t n = t * 16 + in / 32, kw = c * 32 + in % 32;
        out[i] = n < N ? __ldg(q + (n * KW + kw) / 4) : make_uint4(0u, 0u, 0u, 0u);
    }
}

cudaError_t launch_repack(const uint32_t *qweight, int64_t N, int64_t K, uint32_t *out, cudaStream_t stream)
{
    const int64_t threads = (N + 15) / 16 * 16 * (K / 8) / 4;
    const int64_t want = (threads + 255) / 256;
    const unsigned grid = (unsigned)(want < (int64_t)kNumSMs * 16 ? (want > 0 ? want : 1) : (int64_t)kNumSMs * 16);
    return launch_pdl(repack_kernel, dim3(grid), dim3(256), 0, stream, (const uint4 *)qweight, N, K, (uint4 *)out);
}

cudaError_t launch_gemv(const void *X, int64_t M, int64_t N, int64_t K, const uint32_t *qweight,
                        const void *scales, const uint32_t *qzeros, int group, int mode, bool weights_static,
                        bool y_f32, bool repacked, void *Y, cudaStream_t stream)
{
    int *err = device_error_word();
    if (!err) return cudaErrorUnknown;
    CUtensorMap map;
    const cudaError_t e = gemv_code_map(&map, qweight, N, K, repacked);
    if (e != cudaSuccess) return e;
    if (M <= 8)
        return weights_static ? launch_mt<1, true>(map, X, M, N, K, scales, qzeros, group, mode, Y, (y_f32 ? 1 : 0) | (repacked ? 2 : 0), err, stream)
                              : launch_mt<1, false>(map, X, M, N, K, scales, qzeros, group, mode, Y, (y_f32 ? 1 : 0) | (repacked ? 2 : 0), err, stream);
    return weights_static ? launch_mt<2, true>(map, X, M, N, K, scales, qzeros, group, mode, Y, (y_f32 ? 1 : 0) | (repacked ? 2 : 0), err, stream)
                          : launch_mt<2, false>(map, X, M, N, K, scales, qzeros, group, mode, Y, (y_f32 ? 1 : 0) | (repacked ? 2 : 0), err, stream);
}

}  // namespace w4
