// nvfp4_encode.cuh -- the exact NVFP4 block encoder with Four-Over-Six shared by
// the KV-cache quantizer and the weight / activation quantizer: per 16-element
// block, both targets' E4M3 scales from one paired division, E2M1 codes of the
// correctly rounded quotients, and the squared error in the definition's fp32
// order.  Include from files compiled with -fmad=false.
//
// Every function here is one IEEE operation per step of the definition (DeepRead
// page, Method > 训练基础设施: E2M1 values, E4M3 block scale, FP32 tensor scale,
// the block scale searched over targets 6 and 4).
#pragma once

#include "common.cuh"

namespace nvfp4kv {
namespace {

// Markstein's quotient is correctly rounded when no step underflows: the
// tensor scale and the block max are kept above these bounds, else the
// quotient is an IEEE division.
constexpr float kFastMinScale = 0x1p-90f;
constexpr float kFastMinBlockMax = 0x1p-100f;

// L2 eviction policies: inputs read twice are kept (evict_last) on the first
// read and released (evict_first) on the second.
__device__ __forceinline__ uint64_t policy_keep() {
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint64_t policy_release() {
    uint64_t p;
    asm("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
    return p;
}
__device__ __forceinline__ uint4 ld_hint(const uint4* p, uint64_t pol) {
    uint4 r;
    asm("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0,%1,%2,%3}, [%4], %5;"
        : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
        : "l"(p), "l"(pol));
    return r;
}

__device__ __forceinline__ float max_abs8(const float2* x) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(fabsf(x[0].x)), "f"(fabsf(x[0].y)), "f"(fabsf(x[1].x)));
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(d), "f"(fabsf(x[1].y)), "f"(fabsf(x[2].x)));
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(d), "f"(fabsf(x[2].y)), "f"(fabsf(x[3].x)));
    return fmaxf(d, fabsf(x[3].y));
}

// Two bf16 (one word, element 2j low) widened exactly and added to an fp32
// pair, one rounding each: RN(x + c), as two mixed-precision adds on the FMA
// pipe (no separate unpacking).
__device__ __forceinline__ float2 bf16x2_add_f32x2(uint32_t w, float2 c) {
    float lo, hi;
    asm("{.reg .b16 l, h;\n"
        "mov.b32 {l, h}, %2;\n"
        "add.rn.f32.bf16 %0, l, %3;\n"
        "add.rn.f32.bf16 %1, h, %4;}"
        : "=f"(lo), "=f"(hi)
        : "r"(w), "f"(c.x), "f"(c.y));
    return make_float2(lo, hi);
}

// f16 -> f32 (exact) as a mixed-precision add of -0: a full-rate FMA-pipe
// operation, where cvt.f32.f16 issues at half rate.
__device__ __forceinline__ float2 f16x2_to_f32x2(uint32_t h2) {
    float lo, hi;
    asm("{.reg .b16 l, h;\n"
        "mov.b32 {l, h}, %2;\n"
        "add.rn.f32.f16 %0, l, 0f80000000;\n"
        "add.rn.f32.f16 %1, h, 0f80000000;}"
        : "=f"(lo), "=f"(hi)
        : "r"(h2));
    return make_float2(lo, hi);
}

// Four fp32 pairs -> the packed E2M1 codes (byte j = elements 2j, 2j+1) and
// their decoded values as four f16x2, from the same conversion bytes.
__device__ __forceinline__ uint32_t cvt_e2m1x8_dec(const float* v, uint32_t* h) {
    uint32_t r;
    asm("{\n"
        ".reg .b8 b0, b1, b2, b3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %6, %5;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %8, %7;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %10, %9;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %12, %11;\n"
        "cvt.rn.f16x2.e2m1x2 %1, b0;\n"
        "cvt.rn.f16x2.e2m1x2 %2, b1;\n"
        "cvt.rn.f16x2.e2m1x2 %3, b2;\n"
        "cvt.rn.f16x2.e2m1x2 %4, b3;\n"
        "mov.b32 %0, {b0, b1, b2, b3};\n"
        "}"
        : "=r"(r), "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
          "f"(v[7]));
    return r;
}

// Eight elements (four pairs) against one candidate step D with r = RN(1/D):
// packed codes q (byte j = elements 2j, 2j+1) and the sequential sum of the
// eight squared errors RN(RN(x - RN(decode(q) * D))^2).
// The quotient is Markstein's, computed for -x / D so that a zero keeps its
// sign: n0 = RN(x (-r)), e = x + n0 D (exact), n1 = RN(n0 - e r) = -RN(x / D).
// The codes of -x / D are those of x / D with the sign bits flipped (one XOR
// for the stored word); their decoded values dq' = -dq give the error
// directly: RN(x - RN(dq D)) = RN(x + RN(dq' D)).
// The compiler merges a paired product followed by a paired sum into one
// fused multiply-add, which would skip the product's rounding; every sum is
// therefore written as a fused multiply-add whose other factor is 1 held in a
// run-time value (exact, and not mergeable).
__device__ __forceinline__ void encode8_fast(const float2* x, float2 Dr, float one, uint32_t& q,
                                             float& err) {
    const float2 NR = make_float2(-Dr.y, -Dr.y);
    const float2 D2 = make_float2(Dr.x, Dr.x);
    float y[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 n0 = __fmul2_rn(x[j], NR);
        const float2 e = __ffma2_rn(n0, D2, x[j]);
        const float2 n1 = __ffma2_rn(e, NR, n0);
        y[2 * j] = n1.x;
        y[2 * j + 1] = n1.y;
    }
    uint32_t h[4];
    q = cvt_e2m1x8_dec(y, h) ^ 0x88888888u;
    const float2 ONE = make_float2(one, one);
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 p = __fmul2_rn(f16x2_to_f32x2(h[j]), D2);      // RN(dq' D) = -RN(dq D)
        const float2 d = __ffma2_rn(p, ONE, x[j]);                   // RN(x - RN(dq D))
        const float2 sq = __fmul2_rn(d, d);
        acc = (j == 0) ? sq.x : __fmaf_rn(sq.x, one, acc);
        acc = __fmaf_rn(sq.y, one, acc);
    }
    err = acc;
}

// The same with IEEE divisions (tensor scales too small for the fast path);
// out of line, so the rare path costs no instruction-cache space in the loop.
struct Enc8 {
    uint32_t q;
    float err;
};

__device__ __noinline__ Enc8 encode8_slow(float x0, float x1, float x2, float x3, float x4,
                                          float x5, float x6, float x7, float D) {
    const float x[8] = {x0, x1, x2, x3, x4, x5, x6, x7};
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = D > 0.0f ? __fdiv_rn(x[i], D) : 0.0f;
    Enc8 r;
    r.q = cvt_e2m1x8(y);
    uint32_t h[4];
    cvt_e2m1x8_to_f16x2(r.q, h);
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float e0 = __fsub_rn(x[2 * j], __fmul_rn(f16lo(h[j]), D));
        const float e1 = __fsub_rn(x[2 * j + 1], __fmul_rn(f16hi(h[j]), D));
        acc = (j == 0) ? __fmul_rn(e0, e0) : __fadd_rn(acc, __fmul_rn(e0, e0));
        acc = __fadd_rn(acc, __fmul_rn(e1, e1));
    }
    r.err = acc;
    return r;
}

__device__ __noinline__ float2 ratio_slow(float ab, float ms6, float ms4) {
    return make_float2(__fdiv_rn(ab, ms6), __fdiv_rn(ab, ms4));
}

// ---------------------------------------------------------------- Four-Over-Six block encoder
//
// The choice between the two candidates needs their squared errors E6, E4 in
// the definition's fp32 order only when they are close: each candidate's
// error is first estimated cheaply (encode_block16 below), and when the
// estimates are within a threshold several times their error bound, both sums
// are recomputed in the definition's order (sse_exact).  Codes come from the
// correctly rounded quotients either way, so the result is the definition's,
// bit for bit.

// Below this block max the estimate's error analysis (no underflow) is not
// relied on: the exact sums decide.
constexpr float kApproxMinBlockMax = 0x1p-50f;

// The definition's sum for one half block (elements in order): codes q of
// -x / D, step D.  Out of line: it runs only when the estimates are too close.
__device__ __noinline__ float sse_exact(float x0, float x1, float x2, float x3, float x4,
                                        float x5, float x6, float x7, uint32_t q, float D,
                                        float one) {
    const float2 x[4] = {make_float2(x0, x1), make_float2(x2, x3), make_float2(x4, x5),
                         make_float2(x6, x7)};
    uint32_t h[4];
    cvt_e2m1x8_to_f16x2(q, h);
    const float2 D2 = make_float2(D, D);
    const float2 ONE = make_float2(one, one);
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 p = __fmul2_rn(f16x2_to_f32x2(h[j]), D2);      // RN(dq' D) = -RN(dq D)
        const float2 d = __ffma2_rn(p, ONE, x[j]);                   // RN(x - RN(dq D))
        const float2 sq = __fmul2_rn(d, d);
        acc = (j == 0) ? sq.x : __fmaf_rn(sq.x, one, acc);
        acc = __fmaf_rn(sq.y, one, acc);
    }
    return acc;
}

struct EncodeConsts {
    float s, ms6, ms4;
    float2 rm;
    bool fast;
};

__device__ __forceinline__ EncodeConsts encode_consts(float s) {
    EncodeConsts c;
    c.s = s;
    c.ms6 = __fmul_rn(6.0f, s);
    c.ms4 = __fmul_rn(4.0f, s);
    c.rm = make_float2(__frcp_rn(c.ms6), __frcp_rn(c.ms4));
    c.fast = s >= kFastMinScale;
    return c;
}

// ---------------------------------------------------------------- one lane per block
//
// The same encoder with a whole 16-element block in one lane (no shuffles,
// the block-level work done once).  The error estimate is taken in quotient
// units: with y = RN(-x / D) (Markstein, as above) and dq the decoded code of
// x / D, d = RN(dq + y) is one mixed-precision add per element, and
// E' = RN(D^2) * (sum of d^2, fused multiply-adds on pairs).  Its distance from
// the definition's sum E is at most 48 u S + 4 u ab^2 (u = 2^-24, S the exact
// sum of the real errors e, ab the block max): d D = -(e + x eps1)(1 + eps2)
// gives |d^2 D^2 - e^2| <= 2u |e| |x| + 2u e^2 per element, sum |e| |x| <=
// ab^2 + 4 S, and the pair sums, the final add and the scaling by D^2 add
// 10 u S; E itself is within 2u ab^2 + 28 u S of S by the same counting.  The
// threshold below is the two-lane encoder's, 2^-16 (E4' + E6') + 2^-18 ab^2,
// more than twice the bound for both candidates together.

// Two f16 (one word, element 2j low) widened exactly and added to an fp32
// pair, one rounding each: RN(h + c).
__device__ __forceinline__ float2 f16x2_add_f32x2(uint32_t h2, float2 c) {
    float lo, hi;
    asm("{.reg .b16 l, h;\n"
        "mov.b32 {l, h}, %2;\n"
        "add.rn.f32.f16 %0, l, %3;\n"
        "add.rn.f32.f16 %1, h, %4;}"
        : "=f"(lo), "=f"(hi)
        : "r"(h2), "f"(c.x), "f"(c.y));
    return make_float2(lo, hi);
}

// Eight elements against one candidate (D, r = RN(1/D)): the packed codes of
// x / D (byte j = elements 2j, 2j+1) from Markstein's quotients of -x / D,
// and the squared quotient-domain residuals added into acc.
__device__ __forceinline__ uint32_t cand8(const float2* x, float2 Dr, float2& acc) {
    const float2 NR = make_float2(-Dr.y, -Dr.y);
    const float2 D2 = make_float2(Dr.x, Dr.x);
    float2 y[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 n0 = __fmul2_rn(x[j], NR);
        const float2 e = __ffma2_rn(n0, D2, x[j]);
        y[j] = __ffma2_rn(e, NR, n0);                    // -RN(x / D)
    }
    const float yv[8] = {y[0].x, y[0].y, y[1].x, y[1].y, y[2].x, y[2].y, y[3].x, y[3].y};
    const uint32_t q = cvt_e2m1x8(yv) ^ 0x88888888u;     // codes of x / D
    uint32_t h[4];
    cvt_e2m1x8_to_f16x2(q, h);                           // dq
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float2 d = f16x2_add_f32x2(h[j], y[j]);    // RN(dq - x / D)
        acc = __ffma2_rn(d, d, acc);
    }
    return q;
}

struct BlockCodes16 {
    uint2 q;          // codes of elements 0..7, 8..15
    uint32_t sb;
};

// One 16-element block in this lane (x: 8 pairs, ab = max |x|).  The whole
// warp calls it together (the rare exact path is decided warp-wide).
__device__ __forceinline__ BlockCodes16 encode_block16(const float2* x, float ab,
                                                       const float2* tab,
                                                       const EncodeConsts& c, float one) {
    float2 rat;
    if (c.fast && ab >= kFastMinBlockMax) {
        const float2 AB = make_float2(ab, ab);
        const float2 q0 = __fmul2_rn(AB, c.rm);
        const float2 e = __ffma2_rn(q0, make_float2(-c.ms6, -c.ms4), AB);
        rat = __ffma2_rn(e, c.rm, q0);
    } else {
        rat = ratio_slow(ab, c.ms6, c.ms4);
    }
    const uint32_t sbp = cvt_e4m3x2(rat.x, rat.y);
    const uint32_t sb6 = sbp & 0xFFu, sb4 = sbp >> 8;
    const float2 t6 = tab[sb6], t4 = tab[sb4];
    uint2 q6, q4;
    bool keep4;
    if (c.fast) {
        float2 a6 = make_float2(0.0f, 0.0f), a4 = make_float2(0.0f, 0.0f);
        q6.x = cand8(x, t6, a6);
        q6.y = cand8(x + 4, t6, a6);
        q4.x = cand8(x, t4, a4);
        q4.y = cand8(x + 4, t4, a4);
        const float E6 = __fmul_rn(__fmul_rn(t6.x, t6.x), __fadd_rn(a6.x, a6.y));
        const float E4 = __fmul_rn(__fmul_rn(t4.x, t4.x), __fadd_rn(a4.x, a4.y));
        const float diff = __fsub_rn(E4, E6);
        const float tau = __fmaf_rn(0x1p-16f, __fadd_rn(E4, E6), 0x1p-18f * __fmul_rn(ab, ab));
        const bool same = sb6 == sb4;          // identical candidates: equal errors, keep 6
        const bool sure = same || (fabsf(diff) > tau && ab >= kApproxMinBlockMax);
        keep4 = !same && diff < 0.0f;
        if (__any_sync(0xFFFFFFFFu, !sure)) {
            // rare: the definition's sums (elements in order, the halves added)
            const float h6a = sse_exact(x[0].x, x[0].y, x[1].x, x[1].y, x[2].x, x[2].y, x[3].x,
                                        x[3].y, q6.x ^ 0x88888888u, t6.x, one);
            const float h6b = sse_exact(x[4].x, x[4].y, x[5].x, x[5].y, x[6].x, x[6].y, x[7].x,
                                        x[7].y, q6.y ^ 0x88888888u, t6.x, one);
            const float h4a = sse_exact(x[0].x, x[0].y, x[1].x, x[1].y, x[2].x, x[2].y, x[3].x,
                                        x[3].y, q4.x ^ 0x88888888u, t4.x, one);
            const float h4b = sse_exact(x[4].x, x[4].y, x[5].x, x[5].y, x[6].x, x[6].y, x[7].x,
                                        x[7].y, q4.y ^ 0x88888888u, t4.x, one);
            if (!sure) keep4 = __fadd_rn(h4a, h4b) < __fadd_rn(h6a, h6b);
        }
    } else {
        const Enc8 r6a = encode8_slow(x[0].x, x[0].y, x[1].x, x[1].y, x[2].x, x[2].y, x[3].x,
                                      x[3].y, t6.x);
        const Enc8 r6b = encode8_slow(x[4].x, x[4].y, x[5].x, x[5].y, x[6].x, x[6].y, x[7].x,
                                      x[7].y, t6.x);
        const Enc8 r4a = encode8_slow(x[0].x, x[0].y, x[1].x, x[1].y, x[2].x, x[2].y, x[3].x,
                                      x[3].y, t4.x);
        const Enc8 r4b = encode8_slow(x[4].x, x[4].y, x[5].x, x[5].y, x[6].x, x[6].y, x[7].x,
                                      x[7].y, t4.x);
        q6 = make_uint2(r6a.q, r6b.q);
        q4 = make_uint2(r4a.q, r4b.q);
        keep4 = __fadd_rn(r4a.err, r4b.err) < __fadd_rn(r6a.err, r6b.err);
    }
    BlockCodes16 r;
    r.q = keep4 ? q4 : q6;
    if (!((keep4 ? t4.x : t6.x) > 0.0f)) r.q = make_uint2(0u, 0u);   // a zero step stores +0 codes
    r.sb = keep4 ? sb4 : sb6;
    return r;
}

}  // namespace
}  // namespace nvfp4kv
