// w4_quant_pack: fold, group-quantize and pack a bf16 weight matrix.
//
// Method: page 5 (ai-infra.cypggs.com .../02-core-ideas) section 2.2 gives the
// symmetric and asymmetric RTN formulas with round-half-even; page 2
// (learn.longtimenohack.com .../quantization.html) item (1) the groups of g
// weights sharing an fp16 scale and an integer zero-point; page 3
// (blog.freezetheflame.cc quantization deep dive) section 5.3 the offline fold
// W * s.  The exact arithmetic is spelled out in include/w4.h.
//
// Design (HBM-bound stream: 2 B read + about 0.5 B written per weight; the
// SMs' issue budget at full bandwidth is about 11 instructions per weight, so
// the per-weight work is kept to a handful of instructions and the per-group
// work is spread over as many weights as registers allow):
//   * one resident wave of CTAs; the matrix is a row-major sequence of items
//     of 32 lane slices of 64 consecutive weights (2048 weights), and warp w
//     takes items w, w + nwarps, ..., so the warps' shares differ by at most
//     one item; a slice lies in one group (g = 64), in two (g = 32), or in
//     half of one (g = 128: two lanes);
//   * rows of whole slices (K % 64 == 0) are streamed by TMA: each warp keeps
//     two items in flight in a shared-memory ring (a 32-slice x 128-byte box
//     with the 128-byte swizzle, so that a lane's eight 16-byte reads of its
//     slice fall on eight bank groups) and issues the copy of the item after
//     next as soon as its lanes have read an item; other rows are read with
//     four 32-byte loads per lane, the item two steps ahead asked into L2
//     (cp.async.bulk.prefetch);
//   * group amax / min / max: one packed bf16x2 max-of-magnitudes (symmetric)
//     or a min and a max (asymmetric) per raw word (fp32 comparisons after
//     the fold) and at most one __shfl_xor_sync; the per-group IEEE
//     division of the scale and the reciprocal are amortized over 64
//     weights per lane;
//   * with a fold, the 64 weights are folded once per item (w' = fl32(w * s))
//     and kept as fp32 pairs; the smoothing vector is staged once per CTA in
//     shared memory, each 64-factor slice rotated by (slice % 8) float4 so
//     that the lanes' reads of their slices (256 bytes apart) do not collide
//     on banks, and the weights are read past L1 so that it keeps s;
//   * per weight the code is rint(w'/s16) with IEEE semantics (ties to
//     even): t1 = t0 + (w' - t0 * s16) * rcp(s16), t0 = w' * rcp(s16) -- one
//     correction step, the residual exact -- rounds exactly like w'/s16,
//     ties included, for bf16 and folded fp32 weights alike (see quot2), and
//     adding the magic constant 1.5*2^23 leaves 0x4B400000 + rint(t1) in the
//     float's bits (then + zp), two weights per fma/mul/add instruction and
//     no check or fix-up pass.  Groups whose fp16 scale saturated or is
//     subnormal (codes that need clamping) take an IEEE-division path;
//   * the code is monotonic in w', so the asymmetric clamp to [0, 15]
//     (needed before packing: a code of -1 or 16 would borrow from or carry
//     into the next nibble) runs only in warps where some group's extremes
//     map outside;
//   * packing: with bits(y) = C + u (C's low byte 0), one IMAD y_b*16 + y_a
//     puts the byte u_a | u_b << 4 in the low byte; three PRMTs assemble the
//     word (even elements in the low half-word), and each lane stores its 8
//     words as two 16-byte stores;
//   * zero-points of 8 groups are OR-reduced with __shfl_xor_sync across the
//     4, 8 or 16 lanes that hold them and stored once per word.
#include "common.cuh"
#include "tc_ptx.cuh"

#include <cstring>

namespace w4 {
namespace {

// 1.5 * 2^23: for |t| < 2^22, fl32(t + kMagic) has rint(t) in its low mantissa
// bits, because the spacing of floats in [2^23, 2^24) is 1.
constexpr float kMagic = 12582912.0f;
// rcp.approx is within 2 ulp of 1/s16 (quot2 corrects the quotient it gives).
__device__ __forceinline__ float rcp_approx(float d)
{
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(d));
    return r;
}

// 32 bytes of weights.  With STREAM the load does not allocate in L1 (the
// folded path keeps its smoothing factors there instead).
template <bool STREAM>
__device__ __forceinline__ void ld32(const uint4 *p, uint32_t (&v)[8])
{
    if (STREAM)
        asm volatile("ld.global.nc.L1::no_allocate.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                     : "l"(p));
    else
        asm volatile("ld.global.nc.v8.u32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                     : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]), "=r"(v[7])
                     : "l"(p));
}

__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel)
{
    uint32_t d;
    asm("prmt.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
    return d;
}

// One packed word from the magic-added floats of elements 0..7 of an 8-chunk:
// bytes (e0|e2<<4), (e4|e6<<4), (e1|e3<<4), (e5|e7<<4).
__device__ __forceinline__ uint32_t pack_word(const uint32_t *y)
{
    const uint32_t p0 = y[2] * 16u + y[0];
    const uint32_t p1 = y[6] * 16u + y[4];
    const uint32_t p2 = y[3] * 16u + y[1];
    const uint32_t p3 = y[7] * 16u + y[5];
    return prmt(prmt(p0, p1, 0x0040u), prmt(p2, p3, 0x0040u), 0x5410u);
}

__host__ __device__ constexpr int nibble_shift(int e) { return (e & 1) ? 16 + 4 * (e >> 1) : 4 * (e >> 1); }

__device__ __forceinline__ uint32_t bmin2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("min.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

__device__ __forceinline__ uint32_t bmax2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// Per half: the larger of |a| and |b| in magnitude (its sign bit is not used).
__device__ __forceinline__ uint32_t bmaxabs2(uint32_t a, uint32_t b)
{
    uint32_t d;
    asm("max.xorsign.abs.bf16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
    return d;
}

// The quotient x / d (d > 0 an fp16 value, or d = 0 with inv = 0) for rint:
// t0 = fl(x * inv) with inv = rcp.approx(d) (within 2 ulp of 1/d) is within
// |x/d| * 2^-21 of q = x/d; the residual x - t0 * d is a multiple of
// ulp(t0) * ulp(d) below 2^15 of them, so the fma gives it exactly; and
// t1 = fl(t0 + e * inv) is q + (q - t0) * (d * inv - 1) rounded once, i.e.
// within |q| * 2^-42 + half an ulp of q.  For x an fp32 value (a bf16 weight
// or a folded one) and q < 2^11, a half-integer h other than q is farther
// from q than half an ulp of q by at least |q| * 2^-36: x - h * d is a
// nonzero multiple of ulp(x), and ulp(x) / d exceeds half an ulp of q by
// that much because d < 2^(e+1) - ulp(d) for d in [2^e, 2^(e+1)).  So t1 lies
// on q's side of every half-integer, and t1 = h exactly when q = h: rint(t1)
// = rint(q), ties included.
__device__ __forceinline__ float2 quot2(float2 x, float2 inv2, float2 nd2)
{
    const float2 t0 = __fmul2_rn(x, inv2);
    const float2 e = __ffma2_rn(t0, nd2, x);
    return __ffma2_rn(e, inv2, t0);
}

__device__ __forceinline__ float quot(float x, float inv, float d)
{
    const float t0 = __fmul_rn(x, inv);
    const float e = __fmaf_rn(-t0, d, x);
    return __fmaf_rn(e, inv, t0);
}

// The two weights of raw word v (elements 2p and 2p+1 of the lane), folded.
template <bool FOLD>
__device__ __forceinline__ float2 weight_pair(uint32_t v, float2 sp)
{
    const float2 w = make_float2(bf16lo_to_f32(v), bf16hi_to_f32(v));
    return FOLD ? __fmul2_rn(w, sp) : w;
}

// Per-group parameters of the fast path.
struct QParams {
    float inv, magic, d, ymax;
    int zp;
};

// Codes of one 32-weight chunk (16 raw words, or with FOLD the chunk's 16
// folded weight pairs xf, w * s in fp32, and cur is not read): y = fl(t1 +
// magic) holds rint(t1) + zp (or + 8) in its low bits, t1 the corrected
// quotient of quot2, which rounds exactly like w'/s16; for asymmetric groups
// zp is added after the rounding (a tie rounds to even before the shift, as
// rint(w'/s16) + zp asks).  With CLAMP the asymmetric codes are clamped to
// [0, 15] before packing (a code of -1 or 16 would borrow from or carry into
// the neighbouring nibble); without it the caller has shown that every y
// lies in range.  The arithmetic runs on pairs (fma / mul / add of two fp32
// lanes per instruction, each correctly rounded).
template <int MODE, bool FOLD, bool CLAMP>
__device__ __forceinline__ void encode(const uint32_t *cur, const float2 *xf, const QParams &q, uint32_t (&wd)[4])
{
    const float2 inv2 = make_float2(q.inv, q.inv), nd2 = make_float2(-q.d, -q.d);
    const float k = (MODE == W4_SYM) ? q.magic : kMagic;   // + 8 is even: a tie rounds the same way
    const float2 k2 = make_float2(k, k), z2 = make_float2((float)q.zp, (float)q.zp);
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t yb[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = 4 * w + j;
            const float2 x = FOLD ? xf[p] : weight_pair<false>(cur[p], make_float2(1.f, 1.f));
            float2 y = __fadd2_rn(quot2(x, inv2, nd2), k2);
            if (MODE == W4_ASYM) y = __fadd2_rn(y, z2);
            if (MODE == W4_ASYM && CLAMP) {
                y.x = fmaxf(fminf(y.x, q.ymax), kMagic);
                y.y = fmaxf(fminf(y.y, q.ymax), kMagic);
            }
            yb[2 * j] = __float_as_uint(y.x);
            yb[2 * j + 1] = __float_as_uint(y.y);
        }
        wd[w] = pack_word(yb);
    }
}

// The code of one weight by IEEE division (groups whose fp16 scale saturated
// or is subnormal).
template <int MODE>
__device__ __forceinline__ uint32_t division_code(float x, const QParams &q)
{
    const float c = rintf(__fdiv_rn(x, q.d));
    return (MODE == W4_SYM) ? (uint32_t)((int)fminf(fmaxf(c, -8.f), 7.f) + 8)
                            : (uint32_t)(int)fminf(fmaxf(c + (float)q.zp, 0.f), 15.f);
}

// fl32(v / c) for c = 7 or 15 without a division: q0 = v * rc (rc = fl32(1/c)),
// the residual v - q0 * c exactly by an fma, and one correction step.  For
// these two divisors the result is correctly rounded for every one of the 2^23
// significands of a binade, and the steps scale with v over the normal range
// (where the fp16 scale can be nonzero); an infinite v gives NaN, which the
// caller saturates like infinity.
__device__ __forceinline__ float div_const(float v, float c, float rc)
{
    const float q0 = __fmul_rn(v, rc);
    const float r = __fmaf_rn(-q0, c, v);
    return __fmaf_rn(r, rc, q0);
}

// Scale, zero-point and fast-path parameters of a group from the extremes mn
// <= 0 <= mx (asymmetric) or the largest magnitude a (symmetric) of its w'
// (rint(-mn / s16) from quot, like the codes).
template <int MODE>
__device__ __forceinline__ QParams group_params(float a, float mn, float mx, unsigned short &s16, bool &exact_only)
{
    QParams q;
    float s32, hi = 0.f;
    if (MODE == W4_SYM) s32 = div_const(a, 7.0f, __uint_as_float(0x3E124925u));
    else s32 = div_const(__fsub_rn(mx, mn), 15.0f, __uint_as_float(0x3D888889u));
    s16 = !(s32 <= 65504.0f) ? (unsigned short)0x7BFF : __half_as_ushort(__float2half_rn(s32));
    q.d = __half2float(__ushort_as_half(s16));
    q.inv = (q.d > 0.f) ? rcp_approx(q.d) : 0.f;
    if (MODE == W4_SYM) {
        q.zp = 8;
    } else {
        q.zp = (q.d > 0.f) ? (int)fminf(fmaxf(rintf(quot(-mn, q.inv, q.d)), 0.f), 15.f) : 0;
        hi = (float)(15 - q.zp);
    }
    // the fast path assumes a normal, unsaturated fp16 scale (or a zero one)
    exact_only = (s16 == 0x7BFF) || (q.d > 0.f && q.d < 6.103515625e-05f);
    q.magic = kMagic + (float)q.zp;              // exact: 1.5*2^23 + zp < 2^24
    q.ymax = q.magic + hi;
    return q;
}

// The fast path's y (magic + code, before any clamp) of one weight.
template <int MODE>
__device__ __forceinline__ float fast_y(float x, const QParams &q)
{
    const float t = quot(x, q.inv, q.d);
    if (MODE == W4_SYM) return __fadd_rn(t, q.magic);
    return __fadd_rn(__fadd_rn(t, kMagic), (float)q.zp);
}

constexpr int kQItemBytes = 32 * 128;              // one item: 32 slices of 64 bf16
constexpr int kQRingBytes = 8 * 2 * kQItemBytes;   // two items in flight per warp, 8 warps
constexpr int kErrQuantWait = 0x401, kErrQuantDrain = 0x402;

// Bounded wait for an item's copy; false after `limit` ns (an item lands in
// microseconds).
__device__ __noinline__ bool wait_item(uint32_t bar, uint32_t parity, uint64_t limit = kDefaultWaitNs)
{
    uint64_t t0 = 0;
    bool started = false;
    while (true) {
        uint32_t ok;
        asm volatile(
            "{\n\t.reg .pred p;\n\t"
            "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
            "selp.u32 %0, 1, 0, p;\n\t}"
            : "=r"(ok)
            : "r"(bar), "r"(parity)
            : "memory");
        if (ok) return true;
        if (!started) {
            t0 = globaltimer();
            started = true;
        } else if (globaltimer() - t0 > limit) {
            return false;
        }
    }
}

// With TMA (rows whose length is a multiple of 64), each warp streams its
// items into a two-item ring in shared memory: a TMA box of 32 slices x 128
// bytes with the 128-byte swizzle, so that each lane's eight 16-byte reads of
// its own slice hit eight different bank groups; the copy of the item after
// next is issued as soon as the lanes have read an item into registers.
template <int G, int MODE, bool FOLD, bool TMA>
__global__ void __launch_bounds__(256, 2)
quant_pack_kernel(const __grid_constant__ CUtensorMap tmap_w, const uint32_t *__restrict__ W, int N, int K,
                  const float *__restrict__ s, int s_staged, uint4 *__restrict__ qweight,
                  unsigned short *__restrict__ scales, uint32_t *__restrict__ qzeros, int *err, uint64_t wait_ns)
{
    constexpr int GPL = (G == 32) ? 2 : 1;       // groups per lane: a lane owns 64 consecutive weights
    constexpr int LPG = (G == 128) ? 2 : 1;      // lanes per group
    const int lane = threadIdx.x & 31;
    const int warp0 = (int)((blockIdx.x * blockDim.x + threadIdx.x) >> 5);
    const int nwarps = (int)((gridDim.x * blockDim.x) >> 5);
    const int KW = K >> 1;                       // raw words (bf16 pairs) per row
    const int KP = (K + 63) >> 6;                // 64-weight slices per row (the last may hold 32)
    const int NG = K / G, ZW = (NG + 7) >> 3;
    // dynamic shared memory: [TMA: item rings, 1024-aligned; their barriers] then the staged s
    extern __shared__ uint8_t qsm[];
    uint8_t *sbase = TMA ? qsm + ((1024u - (smem_u32(qsm) & 1023u)) & 1023u) : qsm;
    float4 *s_sm = (float4 *)(sbase + (TMA ? kQRingBytes + 1024 : 0));
    const int wib = (int)(threadIdx.x >> 5);     // warp in block
    const uint32_t ring0 = smem_u32(sbase) + wib * 2 * kQItemBytes;
    const uint32_t bar0 = smem_u32(sbase + kQRingBytes) + wib * 16;
    const uint32_t stall_bar = smem_u32(sbase + kQRingBytes) + 256 + wib * 8;   // nothing completes it (failure tests)
    const uint64_t limit = wait_limit_of(wait_ns);
    if (TMA && lane == 0) {
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(bar0 + 8));
        asm volatile("mbarrier.init.shared::cta.b64 [%0], 1;" ::"r"(stall_bar));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        asm volatile("prefetch.tensormap [%0];" ::"l"(&tmap_w) : "memory");
    }
    __syncwarp();
    pdl_wait();                                  // the previous kernel's writes are visible
    pdl_launch_dependents();

    // With a fold and s_staged, the smoothing vector is staged in shared memory
    // once per block: slice c (64 factors, 16 float4) is rotated by c % 8
    // float4, so that the 32 lanes' reads of "their" float4 i hit 8 different
    // 16-byte bank groups (the slices are 256 bytes apart).
    if (FOLD && s_staged) {
        const int n4 = K >> 2, n4p = 16 * ((K + 63) >> 6);   // a half slice at the end is padded with 0
        for (int j = threadIdx.x; j < n4p; j += blockDim.x) {
            const int c = j >> 4, pos = j & 15;
            s_sm[16 * c + ((pos + (c & 7)) & 15)] = j < n4 ? __ldg((const float4 *)s + j) : make_float4(0.f, 0.f, 0.f, 0.f);
        }
        __syncthreads();
    }

    // The work is the row-major sequence of items of 32 slices (2048 weights;
    // the last item of a row may be shorter).  Warp w takes items w,
    // w + nwarps, ... (so every warp gets the same number of items, whatever N
    // and K are) and asks L2 for its items two steps ahead.
    const int IPR = (KP + 31) >> 5;              // items per row
    const int step_rows = nwarps / IPR, step_items = nwarps % IPR;
    auto advance = [&](int &row, int &item) {
        row += step_rows;
        item += step_items;
        if (item >= IPR) {
            item -= IPR;
            ++row;
        }
    };
    auto prefetch_item = [&](int row, int item) {  // lane 0: one item, HBM -> L2
        if (row < N) {
            const int w0 = 1024 * item;
            prefetch_l2(W + (size_t)row * KW + w0, (size_t)min(1024, KW - w0) * 4);
        }
    };
    // lane 0 (TMA): the item (row, item) into ring slot sl
    auto issue = [&](int row, int item, int sl) {
        asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar0 + 8 * sl),
                     "r"(kQItemBytes)
                     : "memory");
        asm volatile(
            "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], "
            "[%2];" ::"r"(ring0 + sl * kQItemBytes),
            "l"(&tmap_w), "r"(bar0 + 8 * sl), "r"(0), "r"(row * KP + 32 * item)
            : "memory");
    };
    int n = warp0 / IPR, it = warp0 % IPR;       // row and item-in-row of the current item
    int pn = n, pit = it;                        // the item two steps ahead
    advance(pn, pit);
    if (lane == 0) {
        if (TMA) {
            if (n < N) issue(n, it, 0);
            if (pn < N) issue(pn, pit, 1);
        } else {
            prefetch_item(n, it);
            prefetch_item(pn, pit);
        }
    }
    advance(pn, pit);

    int j = 0;                                   // items of this warp so far
    bool ok = true;
    while (n < N) {
        if (!TMA && lane == 0) prefetch_item(pn, pit);
        const int cp = 32 * it + lane;           // this lane's slice
        const bool valid = cp < KP;
        const int cpl = valid ? cp : KP - 1;     // a lane past the row end reads the last slice (not stored)
        const bool valid1 = 64 * cpl + 32 < K;   // the slice's second 32-weight chunk is in the row
        const uint32_t *src = W + (size_t)n * KW + 32 * cpl;
        uint32_t cur[32];
        if (TMA) {
            // this lane's slice is row `lane` of the box (a lane past the row end
            // reads the next row's slice, or zeros past the matrix: not stored)
            const int sl = j & 1;
            const bool stall = j == 0 && stalls_first_wait(wait_ns);   // failure-path tests only
            if (!__all_sync(0xffffffffu,
                            wait_item(stall ? stall_bar : bar0 + 8 * sl, stall ? 0u : (uint32_t)(j >> 1) & 1u, limit))) {
                ok = false;
                break;
            }
            const uint8_t *row = sbase + (ring0 - smem_u32(sbase)) + sl * kQItemBytes + lane * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
                const uint4 v = *(const uint4 *)(row + ((c ^ (lane & 7)) << 4));
                cur[4 * c] = v.x;
                cur[4 * c + 1] = v.y;
                cur[4 * c + 2] = v.z;
                cur[4 * c + 3] = v.w;
            }
            __syncwarp();                        // the slot is read: the item after next may land in it
            if (lane == 0 && pn < N) {
                asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
                issue(pn, pit, sl);
            }
        } else {
            ld32<FOLD>((const uint4 *)src, *(uint32_t(*)[8]) & cur[0]);
            ld32<FOLD>((const uint4 *)(src + 8), *(uint32_t(*)[8]) & cur[8]);
            if (valid1) {
                ld32<FOLD>((const uint4 *)(src + 16), *(uint32_t(*)[8]) & cur[16]);
                ld32<FOLD>((const uint4 *)(src + 24), *(uint32_t(*)[8]) & cur[24]);
            } else {
#pragma unroll
                for (int i = 16; i < 32; ++i) cur[i] = 0u;
            }
        }
        advance(pn, pit);
        // with a smoothing fold: the 64 weights w' = fl32(w * s), once per item
        float2 xf[FOLD ? 32 : 1];
        if (FOLD) {
            const float4 *sv = (const float4 *)(s + 64 * (size_t)cpl);
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                float4 f = make_float4(0.f, 0.f, 0.f, 0.f);   // (the missing half of a half slice)
                if (s_staged) f = s_sm[16 * cpl + ((i + (cpl & 7)) & 15)];
                else if (i < 8 || valid1) f = __ldg(sv + i);
                xf[2 * i] = weight_pair<true>(cur[2 * i], make_float2(f.x, f.y));
                xf[2 * i + 1] = weight_pair<true>(cur[2 * i + 1], make_float2(f.z, f.w));
            }
        }

        // ---- group statistics, scales and zero-points ----
        QParams qp[GPL];
        unsigned short s16[GPL];
        bool exact_only = false, clamp = false;
#pragma unroll
        for (int gi = 0; gi < GPL; ++gi) {
            constexpr int WPG = 32 / GPL;        // raw words of the group held by this lane
            float lmin, lmax;                    // extremes of this lane's part of the group (w')
            if (!FOLD && MODE == W4_SYM) {       // on the raw bf16 pairs: one max of magnitudes per pair
                uint32_t pm = cur[WPG * gi];
#pragma unroll
                for (int i = 1; i < WPG; ++i) pm = bmaxabs2(pm, cur[WPG * gi + i]);
                lmin = 0.f;
                lmax = fmaxf(fabsf(bf16lo_to_f32(pm)), fabsf(bf16hi_to_f32(pm)));
            } else if (!FOLD) {                  // one min and one max per pair
                uint32_t pmin = cur[WPG * gi], pmax = cur[WPG * gi];
#pragma unroll
                for (int i = 1; i < WPG; ++i) {
                    pmin = bmin2(pmin, cur[WPG * gi + i]);
                    pmax = bmax2(pmax, cur[WPG * gi + i]);
                }
                lmin = fminf(bf16lo_to_f32(pmin), bf16hi_to_f32(pmin));
                lmax = fmaxf(bf16lo_to_f32(pmax), bf16hi_to_f32(pmax));
            } else if (MODE == W4_SYM) {         // folded: the largest magnitude
                lmin = lmax = 0.f;
#pragma unroll
                for (int i = 0; i < WPG; ++i) {
                    const float2 x = xf[(WPG * gi + i) % (FOLD ? 32 : 1)];
                    lmax = fmaxf(lmax, fmaxf(fabsf(x.x), fabsf(x.y)));
                }
            } else {
                lmin = lmax = 0.f;
#pragma unroll
                for (int i = 0; i < WPG; ++i) {
                    const float2 x = xf[(WPG * gi + i) % (FOLD ? 32 : 1)];
                    lmin = fminf(lmin, fminf(x.x, x.y));
                    lmax = fmaxf(lmax, fmaxf(x.x, x.y));
                }
            }
            float a = 0.f, mn = 0.f, mx = 0.f;
            if (MODE == W4_SYM) {
                a = fmaxf(fabsf(lmin), fabsf(lmax));
                if (LPG == 2) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, 1));
            } else {
                mn = fminf(0.f, lmin);
                mx = fmaxf(0.f, lmax);
                if (LPG == 2) {
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, 1));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
                }
            }
            bool eo;
            qp[gi] = group_params<MODE>(a, mn, mx, s16[gi], eo);
            exact_only |= eo;
            // rint(w'/s16) is monotonic in w', so when the group's extremes map
            // into [0, 15] every weight of the group does and no clamp is needed;
            // symmetric codes never leave [1, 15]: |w'/s16| <= 7 (1 + 2^-11)
            if (MODE == W4_ASYM)
                clamp |= fast_y<MODE>(mn, qp[gi]) < kMagic || fast_y<MODE>(mx, qp[gi]) > qp[gi].ymax;
        }

        // ---- codes ----
        uint32_t wa[4], wb[4];
        if (MODE == W4_ASYM && __any_sync(0xffffffffu, clamp)) {
            encode<MODE, FOLD, true>(cur, xf, qp[0], wa);
            encode<MODE, FOLD, true>(cur + 16, xf + (FOLD ? 16 : 0), qp[GPL - 1], wb);
        } else {
            encode<MODE, FOLD, false>(cur, xf, qp[0], wa);
            encode<MODE, FOLD, false>(cur + 16, xf + (FOLD ? 16 : 0), qp[GPL - 1], wb);
        }
        if (exact_only) {                        // saturated or subnormal scale: IEEE division
#pragma unroll
            for (int w = 0; w < 8; ++w) {
                QParams q = qp[0];
                if (GPL == 2 && w >= 4) q = qp[GPL - 1];
                uint32_t word = 0u;
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 x = FOLD ? xf[(4 * w + e) % (FOLD ? 32 : 1)]
                                          : weight_pair<false>(cur[4 * w + e], make_float2(1.f, 1.f));
                    word |= division_code<MODE>(x.x, q) << nibble_shift(2 * e);
                    word |= division_code<MODE>(x.y, q) << nibble_shift(2 * e + 1);
                }
                if (w < 4) wa[w] = word;
                else wb[w - 4] = word;
            }
        }

        // ---- stores: 2 x 16 bytes of codes, the scales, the zero-points ----
        if (valid) {
            uint4 *dst = qweight + (size_t)n * (K >> 5) + 2 * cp;
            dst[0] = make_uint4(wa[0], wa[1], wa[2], wa[3]);
            if (valid1) dst[1] = make_uint4(wb[0], wb[1], wb[2], wb[3]);
            unsigned short *srow = scales + (size_t)n * NG;
            if (G == 32) {
                srow[2 * cp] = s16[0];
                if (valid1) srow[2 * cp + 1] = s16[GPL - 1];
            } else if (G == 64) {
                srow[cp] = s16[0];
            } else if ((lane & 1) == 0) {
                srow[cp >> 1] = s16[0];
            }
        }
        if (MODE == W4_ASYM) {
            // OR the zero-points of 8 consecutive groups into one word
            uint32_t z = 0u;
            if (G == 32) {
                if (valid) z = ((uint32_t)qp[0].zp << (4 * ((2 * cp) & 7))) |
                               (valid1 ? (uint32_t)qp[GPL - 1].zp << (4 * ((2 * cp + 1) & 7)) : 0u);
            } else if (G == 64) {
                if (valid) z = (uint32_t)qp[0].zp << (4 * (cp & 7));
            } else {
                if (valid && (lane & 1) == 0) z = (uint32_t)qp[0].zp << (4 * ((cp >> 1) & 7));
            }
            constexpr int LPW = (G == 32) ? 4 : (G == 64) ? 8 : 16;   // lanes per zero-point word
#pragma unroll
            for (int off = 1; off < LPW; off <<= 1) z |= __shfl_xor_sync(0xffffffffu, z, off);
            if (valid && (lane & (LPW - 1)) == 0) qzeros[(size_t)n * ZW + cp / LPW] = z;
        }
        advance(n, it);
        ++j;
    }
    if (TMA && !ok && lane == 0) {
        // an item never landed: record it and wait (bounded) for this warp's
        // copies still in flight (items j and j + 1 at most)
        atomicCAS(err, 0, kErrQuantWait);
        int dn = n, dit = it;
        for (int k = j; k < j + 2 && dn < N; ++k) {
            if (!wait_item(bar0 + 8 * (k & 1), (uint32_t)(k >> 1) & 1u)) atomicCAS(err, 0, kErrQuantDrain);
            advance(dn, dit);
        }
    }
}

constexpr int kMaxStagedS = 64 * 1024;          // bytes of smoothing factors staged in shared memory

template <int G, int MODE, bool FOLD, bool TMA>
cudaError_t launch_variant(const CUtensorMap &map, const void *W, int64_t N, int64_t K, const float *s, int staged,
                           size_t smem, uint32_t *qweight, void *scales, uint32_t *qzeros, int *err,
                           cudaStream_t stream)
{
    const int threads = 256;
    static std::atomic<bool> attr_done[kMaxDevices];   // the attribute is per device
    {
        const cudaError_t e =
            set_smem_attr(quant_pack_kernel<G, MODE, FOLD, TMA>, 2048 + kQRingBytes + kMaxStagedS, attr_done);
        if (e != cudaSuccess) return e;
    }
    int per_sm = 0;                              // resident blocks per SM at this shared-memory size
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_pack_kernel<G, MODE, FOLD, TMA>, threads, smem) !=
            cudaSuccess ||
        per_sm < 1)
        per_sm = 1;
    const int64_t items = N * ((K / 64 + 1 + 31) / 32);   // 2048-weight items (upper bound)
    int64_t blocks = (items + 7) / 8;            // one warp per item at most
    const int64_t cap = (int64_t)kNumSMs * per_sm;   // one resident wave; warps stride over rows
    if (blocks > cap) blocks = cap;
    return launch_pdl(quant_pack_kernel<G, MODE, FOLD, TMA>, dim3((unsigned)blocks), dim3(threads), smem, stream, map,
                      (const uint32_t *)W, (int)N, (int)K, s, staged, (uint4 *)qweight, (unsigned short *)scales,
                      qzeros, err, wait_limit_ns());
}

template <int G, int MODE>
cudaError_t launch_g_mode(const void *W, int64_t N, int64_t K, const float *s, uint32_t *qweight, void *scales,
                          uint32_t *qzeros, cudaStream_t stream)
{
    int *err = device_error_word();
    if (!err) return cudaErrorUnknown;
    // TMA for rows of whole 64-weight slices: W as [N K / 64 slices][64 bf16]
    CUtensorMap map;
    memset(&map, 0, sizeof(map));
    bool tma = (K % 64 == 0) && N * (K / 64) <= (int64_t)INT32_MAX && ((uintptr_t)W % 16) == 0;
    if (tma) {
        EncodeTiledFn enc = encode_fn();
        const cuuint64_t gdim[2] = {64u, (cuuint64_t)(N * (K / 64))};
        const cuuint64_t gstride[1] = {128u};
        const cuuint32_t box[2] = {64u, 32u};
        const cuuint32_t estride[2] = {1u, 1u};
        tma = enc && enc(&map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(W), gdim, gstride, box, estride,
                         CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
    }
    const size_t ring = tma ? (size_t)1024 + kQRingBytes + 1024 : 0;   // alignment slack, rings, barriers
    if (s) {
        // the smoothing vector in shared memory when it fits in 64 KB
        const size_t sbytes = (size_t)((K + 63) / 64) * 256;   // whole 64-factor slices
        const int staged = (sbytes <= (size_t)kMaxStagedS) ? 1 : 0;
        const size_t smem = ring + (staged ? sbytes : 0);
        if (tma)
            return launch_variant<G, MODE, true, true>(map, W, N, K, s, staged, smem, qweight, scales, qzeros, err,
                                                       stream);
        return launch_variant<G, MODE, true, false>(map, W, N, K, s, staged, smem, qweight, scales, qzeros, err,
                                                    stream);
    }
    if (tma)
        return launch_variant<G, MODE, false, true>(map, W, N, K, nullptr, 0, ring, qweight, scales, qzeros, err,
                                                    stream);
    return launch_variant<G, MODE, false, false>(map, W, N, K, nullptr, 0, 0, qweight, scales, qzeros, err, stream);
}

}  // namespace

cudaError_t launch_quant_pack(const void *W, int64_t N, int64_t K, int group, int mode, const float *s,
                              uint32_t *qweight, void *scales, uint32_t *qzeros, cudaStream_t stream)
{
    switch (group * 2 + mode) {
    case 32 * 2 + W4_SYM: return launch_g_mode<32, W4_SYM>(W, N, K, s, qweight, scales, qzeros, stream);
    case 32 * 2 + W4_ASYM: return launch_g_mode<32, W4_ASYM>(W, N, K, s, qweight, scales, qzeros, stream);
    case 64 * 2 + W4_SYM: return launch_g_mode<64, W4_SYM>(W, N, K, s, qweight, scales, qzeros, stream);
    case 64 * 2 + W4_ASYM: return launch_g_mode<64, W4_ASYM>(W, N, K, s, qweight, scales, qzeros, stream);
    case 128 * 2 + W4_SYM: return launch_g_mode<128, W4_SYM>(W, N, K, s, qweight, scales, qzeros, stream);
    case 128 * 2 + W4_ASYM: return launch_g_mode<128, W4_ASYM>(W, N, K, s, qweight, scales, qzeros, stream);
    default: return cudaErrorInvalidValue;
    }
}

}  // namespace w4
