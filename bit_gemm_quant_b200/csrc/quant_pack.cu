// w4_quant_pack: fold, group-quantize and pack a bf16 weight matrix.
//
// Method: page 5 (ai-infra.cypggs.com .../02-core-ideas) section 2.2 gives the
// symmetric and asymmetric RTN formulas with round-half-even; page 2
// (learn.longtimenohack.com .../quantization.html) item (1) the groups of g
// weights sharing an fp16 scale and an integer zero-point; page 3
// (blog.freezetheflame.cc quantization deep dive) section 5.3 the offline fold
// W * s.  The exact arithmetic is spelled out in include/w4.h.
//
// Design (HBM-bound stream: 2 B read + about 0.5 B written per weight, a
// budget of roughly 0.4 warp instructions per weight at full bandwidth):
//   * one resident wave of CTAs; warp w quantizes rows w, w + nwarps, ... as a
//     stream of 1024-weight items and loads the next item (across row ends)
//     before it processes the current one; a lane owns 32 consecutive weights,
//     which always lie in one group (g = 32, 64, 128 is 1, 2 or 4 lanes), read
//     with two 32-byte loads; when a warp starts a row it asks L2 to fetch
//     its next row (cp.async.bulk.prefetch), so HBM latency overlaps a whole
//     row of work;
//   * group amax / min / max: 32 in-lane comparisons and at most two
//     __shfl_xor_sync steps; the per-group IEEE divisions (scale and zero
//     point) and the reciprocal are then amortized over 32 weights per lane;
//   * per weight the code is rint(w'/s16) with IEEE semantics: the quotient
//     is approximated as t = w' * rcp(s16); adding the magic constant
//     1.5*2^23 + zp leaves 0x4B400000 + u in the float's bits.  If every t of
//     the lane is further than 2^-16 from a half-integer (the approximation
//     error is below 5 * 2^-20) those codes equal the codes of the exact
//     quotient (a lane takes the exact path with probability ~1e-3);
//     otherwise the lane recomputes its 32 codes with correctly rounded
//     division (__fdiv_rn).  No lower clamp is needed (the group minimum maps
//     to -zp exactly) and in symmetric mode no clamp at all (|t| <= 7 * (1 +
//     2^-11)); groups whose fp16 scale saturated or is subnormal take the
//     exact path;
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

template <int G, int MODE, bool FOLD>
__global__ void __launch_bounds__(256, 3)
quant_pack_kernel(const uint4 *__restrict__ W, int64_t N, int64_t K, const float4 *__restrict__ s,
                  uint4 *__restrict__ qweight, unsigned short *__restrict__ scales, uint32_t *__restrict__ qzeros)
{
    constexpr int LPG = G / 32;                 // lanes per group
    __shared__ uint4 stash[256 * 4];            // 64 bytes per thread, used only to fix flagged codes
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t KC = K >> 5;                  // 32-weight chunks per row
    const int64_t NG = K / G;                   // groups per row
    const int64_t ZW = (NG + 7) >> 3;           // zero-point words per row

    // The warp's work is the stream of (row, 1024-weight chunk) items of rows
    // warp0, warp0 + nwarps, ...; the next item is loaded before the current
    // one is processed, across row boundaries.
    int64_t n = warp0, c0 = 0;
    uint32_t cur[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
    if (n < N && lane < KC) {
        const uint4 *p = W + n * (K >> 3) + 4 * lane;
        ld32(p, *(uint32_t(*)[8])&cur[0]);
        ld32(p + 2, *(uint32_t(*)[8])&cur[8]);
    }
    while (n < N) {
        int64_t nn = n, nc0 = c0 + 32;
        if (nc0 >= KC) { nc0 = 0; nn += nwarps; }
        uint32_t nxt[16] = {0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u, 0u};
        if (nn < N && nc0 + lane < KC) {
            const uint4 *p = W + nn * (K >> 3) + 4 * (nc0 + lane);
            ld32(p, *(uint32_t(*)[8])&nxt[0]);
            ld32(p + 2, *(uint32_t(*)[8])&nxt[8]);
        }
        if (c0 == 0 && lane == 0 && n + nwarps < N)   // the row after this one, HBM -> L2
            prefetch_l2(W + (n + nwarps) * (K >> 3), (size_t)K * 2);
        {
            const int64_t c = c0 + lane;        // this lane's chunk
            const bool valid = c < KC;
            {   // this lane's raw words, for the rare exact fix below
                uint4 *slot = stash + threadIdx.x * 4;
                slot[0] = make_uint4(cur[0], cur[1], cur[2], cur[3]);
                slot[1] = make_uint4(cur[4], cur[5], cur[6], cur[7]);
                slot[2] = make_uint4(cur[8], cur[9], cur[10], cur[11]);
                slot[3] = make_uint4(cur[12], cur[13], cur[14], cur[15]);
            }
            float x[32];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
                const uint32_t v = valid ? cur[i] : 0u;
                x[2 * i] = bf16lo_to_f32(v);
                x[2 * i + 1] = bf16hi_to_f32(v);
            }
            if (FOLD && valid) {                // w' = fl32(w * s[k])
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float4 f = __ldg(s + 8 * c + i);
                    x[4 * i] = __fmul_rn(x[4 * i], f.x);
                    x[4 * i + 1] = __fmul_rn(x[4 * i + 1], f.y);
                    x[4 * i + 2] = __fmul_rn(x[4 * i + 2], f.z);
                    x[4 * i + 3] = __fmul_rn(x[4 * i + 3], f.w);
                }
            }

            // ---- group statistics, scale and zero-point ----
            float d, inv, magic, hi = 0.f;
            int zp;
            unsigned short s16;
            bool exact_only;
            if (MODE == W4_SYM) {
                float a = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) a = fmaxf(a, fabsf(x[i]));
#pragma unroll
                for (int off = LPG / 2; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
                const float s32 = __fdiv_rn(a, 7.0f);
                s16 = (s32 > 65504.0f) ? (unsigned short)0x7BFF : __half_as_ushort(__float2half_rn(s32));
                d = __half2float(__ushort_as_half(s16));
                zp = 8;
            } else {
                float mn = 0.f, mx = 0.f;
#pragma unroll
                for (int i = 0; i < 32; ++i) { mn = fminf(mn, x[i]); mx = fmaxf(mx, x[i]); }
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
            exact_only = (s16 == 0x7BFF) || (d > 0.f && d < 6.103515625e-05f);
            inv = (d > 0.f) ? rcp_approx(d) : 0.f;
            magic = kMagic + (float)zp;         // exact: 1.5*2^23 + zp < 2^24

            // ---- codes ----
            // y = fl(w' * rcp(s16) + (1.5*2^23 + zp)) holds r + zp (or r + 8) in its low
            // bits, r = rint of the approximate quotient.  rho = w' - r*s16 is exact
            // (Sterbenz; r*s16 has <= 16 bits), so |rho| >= s16/2 flags exactly the
            // weights whose code needs the exact decision: ties of the exact quotient
            // (frequent with bf16 weights and short fp16 scales) and roundings the
            // approximation got wrong.  Those are fixed below, one element index at a
            // time, only when some lane of the warp has one.
            const float hd = (d > 0.f) ? 0.5f * d : __int_as_float(0x7F800000);
            // asymmetric codes are clamped to [0, 15] before packing: a code of -1 (a
            // weight at the group minimum whose quotient is a tie below -zp) would
            // borrow from its neighbour nibble in pack_word.  The clamp changes no
            // result: rint(min/s16) = -zp unless zp was clipped to 15, and the method
            // clips every code to [0, 15] anyway.
            const float ymax = magic + hi;
            uint32_t wd[4], flags = 0u;
#pragma unroll
            for (int w = 0; w < 4; ++w) {
                uint32_t yb[8];
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    float y = __fmaf_rn(x[8 * w + i], inv, magic);
                    if (MODE == W4_ASYM) y = fmaxf(fminf(y, ymax), kMagic);
                    const float r = __fsub_rn(y, magic);
                    const float rho = __fmaf_rn(-r, d, x[8 * w + i]);
                    flags |= (fabsf(rho) >= hd) ? (1u << (8 * w + i)) : 0u;
                    yb[i] = __float_as_uint(y);
                }
                wd[w] = pack_word(yb);
            }
            if (__any_sync(0xffffffffu, flags != 0u)) {
                // rare path: fix the flagged codes one by one from the raw bf16 words
                // parked in this lane's shared-memory slot (no live fp32 copies)
                const uint32_t *raw = (const uint32_t *)(stash + threadIdx.x * 4);
                uint32_t m = flags;
                while (m) {
                    const int i = __ffs(m) - 1;
                    m &= m - 1u;
                    float xi = (i & 1) ? bf16hi_to_f32(raw[i >> 1]) : bf16lo_to_f32(raw[i >> 1]);
                    if (FOLD) xi = __fmul_rn(xi, __ldg((const float *)s + 32 * c + i));
                    float y = __fmaf_rn(xi, inv, magic);
                    if (MODE == W4_ASYM) y = fmaxf(fminf(y, ymax), kMagic);
                    const float r = __fsub_rn(y, magic);
                    const float rho = __fmaf_rn(-r, d, xi);
                    // beyond half a step, or an exact tie with r odd: one step toward rho
                    const int odd = (int)(__float_as_uint(y) ^ (uint32_t)zp) & 1;
                    int q = (int)r;
                    if (fabsf(rho) > hd || odd) q += (rho > 0.f) ? 1 : -1;
                    const int u = (MODE == W4_SYM) ? min(max(q, -8), 7) + 8 : min(max(q + zp, 0), 15);
                    const int e = i & 7, sh = (e & 1) ? 16 + 4 * (e >> 1) : 4 * (e >> 1);
                    const uint32_t keep = ~(0xFu << sh), val = (uint32_t)u << sh;
                    const int w = i >> 3;
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
                for (int i = 0; i < 32; ++i) {
                    const float q = rintf(__fdiv_rn(x[i], d));
                    int u;
                    if (MODE == W4_SYM) u = (int)fminf(fmaxf(q, -8.f), 7.f) + 8;
                    else u = (int)fminf(fmaxf(q + (float)zp, 0.f), 15.f);
                    wx[i >> 3] |= (uint32_t)u << nibble_shift(i & 7);
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
        c0 = nc0;
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
    int64_t blocks = (N + 7) / 8;                // one warp per row at most
    const int64_t cap = (int64_t)kNumSMs * per_sm;   // one resident wave; warps stride over rows
    if (blocks > cap) blocks = cap;
    if (s)
        quant_pack_kernel<G, MODE, true><<<(unsigned)blocks, threads, 0, stream>>>(
            (const uint4 *)W, N, K, (const float4 *)s, (uint4 *)qweight, (unsigned short *)scales, qzeros);
    else
        quant_pack_kernel<G, MODE, false><<<(unsigned)blocks, threads, 0, stream>>>(
            (const uint4 *)W, N, K, nullptr, (uint4 *)qweight, (unsigned short *)scales, qzeros);
    return cudaGetLastError();
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
