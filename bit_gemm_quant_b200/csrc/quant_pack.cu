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
// the per-weight work is kept to a handful of instructions):
//   * one resident wave of CTAs; the matrix is a row-major sequence of
//     1024-weight items and warp w takes items w, w + nwarps, ..., so the
//     warps' shares differ by at most one item; a warp loads its next item
//     before it processes the current one and asks L2 for the one after
//     (cp.async.bulk.prefetch); a lane owns 32 consecutive weights, which
//     always lie in one group (g = 32, 64, 128 is 1, 2 or 4 lanes), read with
//     two 32-byte loads;
//   * group amax / min / max: packed bf16x2 min and max over the lane's raw
//     words (fp32 comparisons after the fold) and at most two
//     __shfl_xor_sync steps; the per-group IEEE divisions (scale and zero
//     point) and the reciprocal are amortized over 32 weights per lane;
//   * per weight the code is rint(w'/s16) with IEEE semantics.  The fast path
//     adds the magic constant 1.5*2^23 + zp to w' * rcp(s16), which leaves
//     0x4B400000 + u in the float's bits, and computes the exact residual
//     rho = w' - r * s16 (Sterbenz: r * s16 has <= 16 significant bits), two
//     weights per fma/add instruction.  A pair whose |rho| reaches s16/2 -- an
//     exact tie of the quotient (common with bf16 weights) or a rounding the
//     approximation got wrong -- is flagged and recomputed exactly from the
//     raw words parked in shared memory (ties to even); groups whose fp16
//     scale saturated or is subnormal take an IEEE-division path;
//   * y is monotonic in w', so the asymmetric clamp to [0, 15] (needed before
//     packing: a code of -1 or 16 would borrow from or carry into the next
//     nibble) runs only in warps where some group's extremes map outside;
//   * packing: with bits(y) = C + u (C's low byte 0), one IMAD y_b*16 + y_a
//     puts the byte u_a | u_b << 4 in the low byte; three PRMTs assemble the
//     word (even elements in the low half-word), and each lane stores its 4
//     words as one 16-byte store (a warp writes 512 contiguous bytes);
//   * zero-points of 8 groups are OR-reduced with __shfl_xor_sync inside their
//     8*g/32-lane segment and stored once per word.
#include "common.cuh"

namespace w4 {
namespace {

// 1.5 * 2^23: for |t| < 2^22, fl32(t + kMagic) has rint(t) in its low mantissa
// bits, because the spacing of floats in [2^23, 2^24) is 1.
constexpr float kMagic = 12582912.0f;
// rcp.approx is within 2 ulp of 1/s16, so w' * rcp(s16) is within
// |w'/s16| * 2^-22 <= 2^-18 of the exact quotient: a rounding it gets wrong
// leaves a residual of at least half a step, which the exact check catches.
__device__ __forceinline__ float rcp_approx(float d)
{
    float r;
    asm("rcp.approx.f32 %0, %1;" : "=f"(r) : "f"(d));
    return r;
}

__device__ __forceinline__ void ld32(const uint4 *p, uint32_t (&v)[8])
{
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

// The two weights of raw word v (elements 2p and 2p+1 of the lane), folded.
template <bool FOLD>
__device__ __forceinline__ float2 weight_pair(uint32_t v, float2 sp)
{
    const float2 w = make_float2(bf16lo_to_f32(v), bf16hi_to_f32(v));
    return FOLD ? __fmul2_rn(w, sp) : w;
}

// Fast-path codes of the lane's 32 weights: y = fl(w' * rcp(s16) + magic)
// holds r + zp (or r + 8) in its low bits, r = rint of the approximate
// quotient; rho = w' - r * s16 is exact.  Bit p of the returned flags marks the
// weight pair p if either residual reaches half a step (|rho| >= s16 / 2):
// exact ties of the quotient and roundings the approximation got wrong.  With
// CLAMP the asymmetric codes are clamped to [0, 15] before packing (a code of
// -1 or 16 would borrow from or carry into the neighbouring nibble); without
// it the caller has shown that every y lies in range.  The arithmetic runs on
// pairs (fma / add of two fp32 lanes per instruction, each correctly rounded).
template <int MODE, bool FOLD, bool CLAMP>
__device__ __forceinline__ uint32_t encode(const uint32_t (&cur)[16], const float2 (&sp)[16], float inv,
                                           float magic, float d, float hd, float ymax, uint32_t (&wd)[4])
{
    const float2 inv2 = make_float2(inv, inv), mg2 = make_float2(magic, magic);
    const float2 nmg2 = make_float2(-magic, -magic), nd2 = make_float2(-d, -d);
    uint32_t flags = 0u;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
        uint32_t yb[8];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            const int p = 4 * w + j;
            const float2 x = weight_pair<FOLD>(cur[p], sp[p]);
            float2 y = __ffma2_rn(x, inv2, mg2);
            if (MODE == W4_ASYM && CLAMP) {
                y.x = fmaxf(fminf(y.x, ymax), kMagic);
                y.y = fmaxf(fminf(y.y, ymax), kMagic);
            }
            const float2 r = __fadd2_rn(y, nmg2);
            const float2 rho = __ffma2_rn(r, nd2, x);
            if (fmaxf(fabsf(rho.x), fabsf(rho.y)) >= hd) flags |= 1u << p;
            yb[2 * j] = __float_as_uint(y.x);
            yb[2 * j + 1] = __float_as_uint(y.y);
        }
        wd[w] = pack_word(yb);
    }
    return flags;
}

// The exact code of one weight (its fast-path y recomputed, then the tie or
// the wrong rounding resolved from the exact residual).
template <int MODE>
__device__ __forceinline__ uint32_t exact_code(float x, float inv, float magic, float d, float hd, float ymax, int zp)
{
    float y = __fmaf_rn(x, inv, magic);
    if (MODE == W4_ASYM) y = fmaxf(fminf(y, ymax), kMagic);
    const float r = __fsub_rn(y, magic);
    const float rho = __fmaf_rn(-r, d, x);
    const float ar = fabsf(rho);
    // beyond half a step, or an exact tie with r odd: one step toward rho
    const int odd = (int)(__float_as_uint(y) ^ (uint32_t)zp) & 1;
    int q = (int)r;
    if (ar > hd || (ar == hd && odd)) q += (rho > 0.f) ? 1 : -1;
    return (MODE == W4_SYM) ? (uint32_t)(min(max(q, -8), 7) + 8) : (uint32_t)min(max(q + zp, 0), 15);
}

template <int G, int MODE, bool FOLD>
__global__ void __launch_bounds__(256, 3)
quant_pack_kernel(const uint4 *__restrict__ W, int64_t N, int64_t K, const float4 *__restrict__ s,
                  uint4 *__restrict__ qweight, unsigned short *__restrict__ scales, uint32_t *__restrict__ qzeros)
{
    constexpr int LPG = G / 32;                 // lanes per group
    __shared__ uint4 stash[4][256];             // raw words, [quarter][thread]: for the rare exact fix
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t KC = K >> 5;                  // 32-weight chunks per row
    const int64_t NG = K / G;                   // groups per row
    const int64_t ZW = (NG + 7) >> 3;           // zero-point words per row
    pdl_wait();                                 // the previous kernel's writes are visible
    pdl_launch_dependents();

    // The work is the row-major sequence of 1024-weight items (32 chunks of a
    // row; the last item of a row may be shorter).  Warp w takes items w,
    // w + nwarps, w + 2 nwarps, ... (so every warp gets the same number of
    // items, whatever N and K), loads its next item before it processes the
    // current one and asks L2 for the item after that.  Lanes past the end of
    // a row keep zero words (they are not stored).
    const int64_t IPR = (KC + 31) >> 5;         // items per row
    const int64_t step_rows = nwarps / IPR, step_items = nwarps % IPR;
    auto advance = [&](int64_t &row, int64_t &item) {
        row += step_rows;
        item += step_items;
        if (item >= IPR) { item -= IPR; ++row; }
    };
    int64_t n = warp0 / IPR, it = warp0 % IPR;  // row and item-in-row of the current item
    uint32_t cur[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (n < N && 32 * it + lane < KC) {
        const uint4 *p = W + n * (K >> 3) + 4 * (32 * it + lane);
        ld32(p, *(uint32_t(*)[8])&cur[0]);
        ld32(p + 2, *(uint32_t(*)[8])&cur[8]);
    }
    while (n < N) {
        const int64_t c0 = 32 * it;             // first chunk of the current item
        int64_t nn = n, nit = it;
        advance(nn, nit);
        uint32_t nxt[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (nn < N && 32 * nit + lane < KC) {
            const uint4 *p = W + nn * (K >> 3) + 4 * (32 * nit + lane);
            ld32(p, *(uint32_t(*)[8])&nxt[0]);
            ld32(p + 2, *(uint32_t(*)[8])&nxt[8]);
        }
        if (lane == 0) {                        // the item after next, HBM -> L2
            int64_t pn = nn, pit = nit;
            advance(pn, pit);
            if (pn < N) {
                const int64_t pc = 32 * pit, nch = (KC - pc) < 32 ? (KC - pc) : 32;
                prefetch_l2(W + pn * (K >> 3) + 4 * pc, (size_t)nch * 64);
            }
        }
        {
            const int64_t c = c0 + lane;        // this lane's chunk
            const bool valid = c < KC;
#pragma unroll
            for (int q = 0; q < 4; ++q)
                stash[q][threadIdx.x] = make_uint4(cur[4 * q], cur[4 * q + 1], cur[4 * q + 2], cur[4 * q + 3]);
            float2 sp[16];                      // smoothing factors of the weight pairs
#pragma unroll
            for (int i = 0; i < 8; ++i) {
                const float4 f = (FOLD && valid) ? __ldg(s + 8 * c + i) : make_float4(1.f, 1.f, 1.f, 1.f);
                sp[2 * i] = make_float2(f.x, f.y);
                sp[2 * i + 1] = make_float2(f.z, f.w);
            }

            // ---- group statistics, scale and zero-point ----
            float lmin, lmax;                   // extremes of this lane's 32 weights w'
            if (!FOLD) {                        // on the raw bf16 pairs: one min and one max per pair
                uint32_t pmin = cur[0], pmax = cur[0];
#pragma unroll
                for (int i = 1; i < 16; ++i) { pmin = bmin2(pmin, cur[i]); pmax = bmax2(pmax, cur[i]); }
                lmin = fminf(bf16lo_to_f32(pmin), bf16hi_to_f32(pmin));
                lmax = fmaxf(bf16lo_to_f32(pmax), bf16hi_to_f32(pmax));
            } else {
                lmin = lmax = 0.f;
#pragma unroll
                for (int i = 0; i < 16; ++i) {
                    const float2 x = weight_pair<true>(cur[i], sp[i]);
                    lmin = fminf(lmin, fminf(x.x, x.y));
                    lmax = fmaxf(lmax, fmaxf(x.x, x.y));
                }
            }
            float d, mn = 0.f, mx = 0.f, hi = 0.f;
            int zp;
            unsigned short s16;
            if (MODE == W4_SYM) {
                float a = fmaxf(fabsf(lmin), fabsf(lmax));
#pragma unroll
                for (int off = LPG / 2; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
                const float s32 = __fdiv_rn(a, 7.0f);
                s16 = (s32 > 65504.0f) ? (unsigned short)0x7BFF : __half_as_ushort(__float2half_rn(s32));
                d = __half2float(__ushort_as_half(s16));
                zp = 8;
            } else {
                mn = fminf(0.f, lmin);
                mx = fmaxf(0.f, lmax);
#pragma unroll
                for (int off = LPG / 2; off > 0; off >>= 1) {
                    mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
                    mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                }
                const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
                s16 = (s32 > 65504.0f) ? (unsigned short)0x7BFF : __half_as_ushort(__float2half_rn(s32));
                d = __half2float(__ushort_as_half(s16));
                zp = (d > 0.f) ? (int)fminf(fmaxf(rintf(__fdiv_rn(-mn, d)), 0.f), 15.f) : 0;
                hi = (float)(15 - zp);
            }
            // the fast path assumes a normal, unsaturated fp16 scale (or a zero one)
            const bool exact_only = (s16 == 0x7BFF) || (d > 0.f && d < 6.103515625e-05f);
            const float inv = (d > 0.f) ? rcp_approx(d) : 0.f;
            const float magic = kMagic + (float)zp;   // exact: 1.5*2^23 + zp < 2^24
            const float hd = (d > 0.f) ? 0.5f * d : __int_as_float(0x7F800000);
            const float ymax = magic + hi;

            // ---- codes ----
            // y is monotonic in w', so when the group's extremes mn and mx map into
            // [0, 15] every weight of the group does and no clamp is needed; the
            // (rare) warps with a group whose extremes fall outside run the clamped
            // variant.  Symmetric codes never leave [1, 15]: |w'/s16| <= 7 (1 + 2^-11).
            uint32_t wd[4], flags;
            bool clamp = false;
            if (MODE == W4_ASYM)
                clamp = __fmaf_rn(mn, inv, magic) < kMagic || __fmaf_rn(mx, inv, magic) > ymax;
            if (MODE == W4_ASYM && __any_sync(0xffffffffu, clamp))
                flags = encode<MODE, FOLD, true>(cur, sp, inv, magic, d, hd, ymax, wd);
            else
                flags = encode<MODE, FOLD, false>(cur, sp, inv, magic, d, hd, ymax, wd);
            if (__any_sync(0xffffffffu, flags != 0u)) {
                // fix the flagged pairs from the raw words parked in shared memory
                // (a warp has one in about two items with bf16 weights: exact ties
                // are common when the fp16 scale has few significant bits)
                uint32_t m = flags;
                while (m) {
                    const int p = __ffs(m) - 1;
                    m &= m - 1u;
                    const uint32_t v = ((const uint32_t *)&stash[p >> 2][threadIdx.x])[p & 3];
                    float2 sv = make_float2(1.f, 1.f);
                    if (FOLD) sv = __ldg((const float2 *)s + 16 * c + p);
                    const float2 x = weight_pair<FOLD>(v, sv);
                    const uint32_t u0 = exact_code<MODE>(x.x, inv, magic, d, hd, ymax, zp);
                    const uint32_t u1 = exact_code<MODE>(x.y, inv, magic, d, hd, ymax, zp);
                    // elements 2p, 2p+1: nibble (p & 3) of the low and of the high half-word
                    const int sh = 4 * (p & 3), w = p >> 2;
                    const uint32_t keep = ~((0xFu << sh) | (0xFu << (16 + sh)));
                    const uint32_t val = (u0 << sh) | (u1 << (16 + sh));
                    wd[0] = (w == 0) ? ((wd[0] & keep) | val) : wd[0];
                    wd[1] = (w == 1) ? ((wd[1] & keep) | val) : wd[1];
                    wd[2] = (w == 2) ? ((wd[2] & keep) | val) : wd[2];
                    wd[3] = (w == 3) ? ((wd[3] & keep) | val) : wd[3];
                }
            }
            uint4 out = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            if (exact_only) {                   // saturated or subnormal scale: IEEE division
                uint32_t wx[4] = {0u, 0u, 0u, 0u};
#pragma unroll
                for (int p = 0; p < 16; ++p) {
                    const float2 x = weight_pair<FOLD>(cur[p], sp[p]);
#pragma unroll
                    for (int h = 0; h < 2; ++h) {
                        const float q = rintf(__fdiv_rn(h ? x.y : x.x, d));
                        int u;
                        if (MODE == W4_SYM) u = (int)fminf(fmaxf(q, -8.f), 7.f) + 8;
                        else u = (int)fminf(fmaxf(q + (float)zp, 0.f), 15.f);
                        wx[p >> 2] |= (uint32_t)u << nibble_shift(2 * (p & 3) + h);
                    }
                }
                out = make_uint4(wx[0], wx[1], wx[2], wx[3]);
            }

            const int64_t j = (c * 32) / G;     // group of this lane
            if (valid) {
                qweight[n * KC + c] = out;      // 16 bytes = the 32 codes of this lane
                if ((lane % LPG) == 0) scales[n * NG + j] = s16;
            }
            if (MODE == W4_ASYM) {
                // OR the zero-points of 8 consecutive groups (8*LPG lanes) into one word
                uint32_t z = (valid && (lane % LPG) == 0) ? ((uint32_t)zp << (4 * (int)(j & 7))) : 0u;
#pragma unroll
                for (int off = 1; off < 8 * LPG; off <<= 1) z |= __shfl_xor_sync(0xffffffffu, z, off);
                if (valid && (lane % (8 * LPG)) == 0) qzeros[n * ZW + (j >> 3)] = z;
            }
        }
#pragma unroll
        for (int i = 0; i < 16; ++i) cur[i] = nxt[i];
        n = nn;
        it = nit;
    }
}

template <int G, int MODE>
cudaError_t launch_g_mode(const void *W, int64_t N, int64_t K, const float *s, uint32_t *qweight, void *scales,
                          uint32_t *qzeros, cudaStream_t stream)
{
    const int threads = 256;
    static int per_sm = 0;                       // resident blocks per SM of this instantiation
    if (per_sm == 0) {
        const cudaError_t e = s ? cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_pack_kernel<G, MODE, true>, threads, 0)
                                : cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quant_pack_kernel<G, MODE, false>, threads, 0);
        if (e != cudaSuccess || per_sm < 1) per_sm = 1;
    }
    const int64_t items = N * ((K / 32 + 31) / 32);   // 1024-weight items
    int64_t blocks = (items + 7) / 8;            // one warp per item at most
    const int64_t cap = (int64_t)kNumSMs * per_sm;   // one resident wave; warps stride over rows
    if (blocks > cap) blocks = cap;
    if (s)
        return launch_pdl(quant_pack_kernel<G, MODE, true>, dim3((unsigned)blocks), dim3(threads), 0, stream,
                          (const uint4 *)W, N, K, (const float4 *)s, (uint4 *)qweight, (unsigned short *)scales,
                          qzeros);
    return launch_pdl(quant_pack_kernel<G, MODE, false>, dim3((unsigned)blocks), dim3(threads), 0, stream,
                      (const uint4 *)W, N, K, (const float4 *)nullptr, (uint4 *)qweight, (unsigned short *)scales,
                      qzeros);
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
