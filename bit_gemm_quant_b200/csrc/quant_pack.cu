// w4_quant_pack: fold, group-quantize and pack a bf16 weight matrix.
//
// Method: page 5 (ai-infra.cypggs.com .../02-core-ideas) section 2.2 gives the
// symmetric and asymmetric RTN formulas with round-half-even; page 2
// (learn.longtimenohack.com .../quantization.html) item (1) the groups of g
// weights sharing an fp16 scale and an integer zero-point; page 3
// (blog.freezetheflame.cc quantization deep dive) section 5.3 the offline fold
// W * s.  The exact arithmetic is spelled out in include/w4.h.
//
// Design (HBM-bound stream: 2 B read + 0.5 B written per weight):
//   * one warp per row at a time (grid-stride over rows); a lane owns 8
//     consecutive weights (one 16-byte load), so a group of g weights is g/8
//     adjacent lanes and its amax / min / max is a butterfly of
//     __shfl_xor_sync over those lanes;
//   * a batch is 4 loads per lane (1024 weights per warp) issued before any
//     arithmetic, so every warp keeps 2 KB in flight;
//   * each lane packs its 8 codes into one 32-bit word (even elements in the
//     low half-word), so a warp stores 128 contiguous bytes per iteration;
//     zero-points of 8 groups are OR-reduced across the warp with
//     __reduce_or_sync and stored once per word;
//   * per element the code is rint(w'/s16) with IEEE semantics: the quotient
//     is first approximated as w' * rcp(s16); when that approximation is
//     further than 2^-10 from every half-integer its rounding cannot differ
//     from that of the exact quotient (the approximation error is below
//     2^-18), so the code is read from the approximation with a magic-number
//     add; otherwise the lane recomputes its 8 codes with correctly rounded
//     division (__fdiv_rn).  Per-group scale and zero-point use __fdiv_rn
//     directly, so both are bit-identical to the IEEE definitions.
#include "common.cuh"

namespace w4 {
namespace {

// 1.5 * 2^23: for |t| < 2^22, fl32(t + kMagic) has rint(t) (ties to even) in
// its low mantissa bits, because the spacing of floats in [2^23, 2^24) is 1.
constexpr float kMagic = 12582912.0f;
// Quotients closer than 2^-10 to a half-integer take the exact path.
constexpr float kNearTie = 0.5f - 0.0009765625f;

__device__ __forceinline__ uint4 ld_stream(const uint4 *p)
{
    uint4 v;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                 : "l"(p));
    return v;
}

// Bit offset of element e (0..7) inside its packed word: even elements in the
// low half-word, odd elements in the high half-word.
__host__ __device__ constexpr int nibble_shift(int e) { return (e & 1) ? 16 + 4 * (e >> 1) : 4 * (e >> 1); }

template <int G, int MODE, bool FOLD>
__global__ void __launch_bounds__(256)
quant_pack_kernel(const uint4 *__restrict__ W, int64_t N, int64_t K, const float4 *__restrict__ s,
                  uint32_t *__restrict__ qweight, unsigned short *__restrict__ scales,
                  uint32_t *__restrict__ qzeros)
{
    constexpr int LPG = G / 8;                  // lanes per group
    constexpr int ZPB = 128 / G;                // zero-point words per 1024-weight batch
    const int lane = threadIdx.x & 31;
    const int64_t warp0 = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
    const int64_t nwarps = ((int64_t)gridDim.x * blockDim.x) >> 5;
    const int64_t KW = K >> 3;                  // packed words (= 16-byte bf16 chunks) per row
    const int64_t NG = K / G;                   // groups per row
    const int64_t ZW = (NG + 7) >> 3;           // zero-point words per row

    for (int64_t n = warp0; n < N; n += nwarps) {
        const uint4 *row = W + n * KW;
        for (int64_t c0 = 0; c0 < KW; c0 += 128) {
            uint4 v[4];
            float4 sa[4], sb[4];
#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int64_t c = c0 + it * 32 + lane;
                if (c < KW) {
                    v[it] = ld_stream(row + c);
                    if (FOLD) { sa[it] = __ldg(s + 2 * c); sb[it] = __ldg(s + 2 * c + 1); }
                } else {
                    v[it] = make_uint4(0u, 0u, 0u, 0u);
                    if (FOLD) { sa[it] = make_float4(1.f, 1.f, 1.f, 1.f); sb[it] = sa[it]; }
                }
            }
            uint32_t zacc[ZPB];
#pragma unroll
            for (int i = 0; i < ZPB; ++i) zacc[i] = 0u;

#pragma unroll
            for (int it = 0; it < 4; ++it) {
                const int64_t c = c0 + it * 32 + lane;
                const bool valid = c < KW;
                float x[8];
                x[0] = bf16lo_to_f32(v[it].x); x[1] = bf16hi_to_f32(v[it].x);
                x[2] = bf16lo_to_f32(v[it].y); x[3] = bf16hi_to_f32(v[it].y);
                x[4] = bf16lo_to_f32(v[it].z); x[5] = bf16hi_to_f32(v[it].z);
                x[6] = bf16lo_to_f32(v[it].w); x[7] = bf16hi_to_f32(v[it].w);
                if (FOLD) {   // w' = fl32(w * s[k])
                    x[0] = __fmul_rn(x[0], sa[it].x); x[1] = __fmul_rn(x[1], sa[it].y);
                    x[2] = __fmul_rn(x[2], sa[it].z); x[3] = __fmul_rn(x[3], sa[it].w);
                    x[4] = __fmul_rn(x[4], sb[it].x); x[5] = __fmul_rn(x[5], sb[it].y);
                    x[6] = __fmul_rn(x[6], sb[it].z); x[7] = __fmul_rn(x[7], sb[it].w);
                }

                float d, inv, lo, hi;
                int zp;
                unsigned short s16;
                if (MODE == W4_SYM) {
                    float a = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) a = fmaxf(a, fabsf(x[i]));
#pragma unroll
                    for (int off = LPG / 2; off > 0; off >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, off));
                    const float s32 = __fdiv_rn(a, 7.0f);
                    s16 = (s32 > 65504.0f) ? (unsigned short)0x7BFF : __half_as_ushort(__float2half_rn(s32));
                    d = __half2float(__ushort_as_half(s16));
                    inv = (d > 0.f) ? __frcp_rn(d) : 0.f;
                    zp = 8;
                    lo = -8.f;
                    hi = 7.f;
                } else {
                    float mn = 0.f, mx = 0.f;
#pragma unroll
                    for (int i = 0; i < 8; ++i) { mn = fminf(mn, x[i]); mx = fmaxf(mx, x[i]); }
#pragma unroll
                    for (int off = LPG / 2; off > 0; off >>= 1) {
                        mn = fminf(mn, __shfl_xor_sync(0xffffffffu, mn, off));
                        mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
                    }
                    const float s32 = __fdiv_rn(__fsub_rn(mx, mn), 15.0f);
                    s16 = (s32 > 65504.0f) ? (unsigned short)0x7BFF : __half_as_ushort(__float2half_rn(s32));
                    d = __half2float(__ushort_as_half(s16));
                    if (d > 0.f) {
                        inv = __frcp_rn(d);
                        zp = (int)fminf(fmaxf(rintf(__fdiv_rn(-mn, d)), 0.f), 15.f);
                    } else {
                        inv = 0.f;
                        zp = 0;
                    }
                    lo = (float)(-zp);
                    hi = (float)(15 - zp);
                }

                // codes: fast path from the approximate quotient
                uint32_t word = 0u;
                bool near_tie = false;
                const float magic = (MODE == W4_SYM) ? kMagic + 8.0f : kMagic;   // both even
#pragma unroll
                for (int i = 0; i < 8; ++i) {
                    const float t = fminf(fmaxf(__fmul_rn(x[i], inv), lo), hi);
                    const float y = __fadd_rn(t, magic);
                    const float r = __fsub_rn(y, magic);
                    near_tie |= fabsf(__fsub_rn(t, r)) > kNearTie;
                    uint32_t u = __float_as_uint(y);
                    if (MODE == W4_ASYM) u += (uint32_t)zp;
                    word |= (u & 0xFu) << nibble_shift(i);
                }
                if (near_tie) {   // exact path: rint of the correctly rounded quotient
                    word = 0u;
#pragma unroll
                    for (int i = 0; i < 8; ++i) {
                        const float q = rintf(__fdiv_rn(x[i], d));
                        int u;
                        if (MODE == W4_SYM) u = (int)fminf(fmaxf(q, -8.f), 7.f) + 8;
                        else u = (int)fminf(fmaxf(q + (float)zp, 0.f), 15.f);
                        word |= (uint32_t)u << nibble_shift(i);
                    }
                }

                const int64_t j = (c * 8) / G;      // group of this lane
                if (valid) {
                    qweight[n * KW + c] = word;
                    if ((lane % LPG) == 0) scales[n * NG + j] = s16;
                }
                if (MODE == W4_ASYM) {
                    const uint32_t mine = (valid && (lane % LPG) == 0) ? ((uint32_t)zp << (4 * (int)(j & 7))) : 0u;
                    zacc[(it * 32) / G] |= __reduce_or_sync(0xffffffffu, mine);
                }
            }
            if (MODE == W4_ASYM) {
#pragma unroll
                for (int i = 0; i < ZPB; ++i) {
                    const int64_t zw = (c0 * 8) / (8 * G) + i;
                    if (lane == i && zw < ZW) qzeros[n * ZW + zw] = zacc[i];
                }
            }
        }
    }
}

template <int G, int MODE>
cudaError_t launch_g_mode(const void *W, int64_t N, int64_t K, const float *s, uint32_t *qweight, void *scales,
                          uint32_t *qzeros, cudaStream_t stream)
{
    const int threads = 256;
    int64_t blocks = (N + 7) / 8;                // one warp per row
    const int64_t cap = (int64_t)kNumSMs * 8;    // grid-stride beyond 8 resident blocks per SM
    if (blocks > cap) blocks = cap;
    if (s)
        quant_pack_kernel<G, MODE, true><<<(unsigned)blocks, threads, 0, stream>>>(
            (const uint4 *)W, N, K, (const float4 *)s, qweight, (unsigned short *)scales, qzeros);
    else
        quant_pack_kernel<G, MODE, false><<<(unsigned)blocks, threads, 0, stream>>>(
            (const uint4 *)W, N, K, nullptr, qweight, (unsigned short *)scales, qzeros);
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
