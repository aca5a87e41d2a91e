// common.cuh -- device helpers shared by the library's kernels: workspace
// control words, a bounded grid barrier, bf16 unpacking and the sm_100
// conversion instructions for the NVFP4 formats.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "nvfp4kv.h"

namespace nvfp4kv {

constexpr int kHeadDim = 128;        // d supported by the kernels
constexpr int kBlock = 16;           // micro-block length along d
constexpr int kSegment = 64;         // K-smoothing partial-sum segment (tokens)
constexpr float kTensorScaleDiv = 2688.0f;   // 6 * 448

// Status bits recorded by kernels in the workspace.
constexpr unsigned kStatusTimeout = 1u;
constexpr unsigned kStatusRange = 2u;   // attention: key set's V scales span more than 2^116

// Time limit of any single wait inside a kernel, in nanoseconds; a wait that
// reaches it records kStatusTimeout (and its site) and the kernel returns.
constexpr unsigned long long kWaitLimitNs = 200ull * 1000 * 1000;

// First 256 bytes of every workspace.
struct Control {
    unsigned status;      // OR of kStatus* bits; cleared by the host
    unsigned bar_count;   // grid barrier: CTAs arrived at the current barrier
    unsigned bar_gen;     // grid barrier: generation, bumped by the last arrival
    unsigned diag[4];     // first wait that gave up: site, block (x | y << 16), step, phase
    unsigned test_flags;  // test hooks, 0 in normal use (bit 0: see attention_ws.cu)
    unsigned pad0;
    unsigned long long stamp[8];   // %globaltimer at CTA 0's phase boundaries (diagnostics)
    // the chunk quantizer's progress across CTAs (its last CTA resets them)
    unsigned q_vdone;     // CTAs whose max |V| is folded into q_vmax
    unsigned q_vmax;      // max |V| (float bits: non-negative floats order as their bits)
    unsigned q_sdone;     // K statistics units written
    unsigned q_fdone;     // 32-column blocks whose mean is written
    unsigned q_kmax;      // max |K - mean| (float bits)
    unsigned q_exit;      // CTAs finished
    unsigned pad[32];
};

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

// Record a wait that gave up: the status bit, and the first such site.
__device__ __forceinline__ void record_timeout(Control* ctl, unsigned site, unsigned step,
                                               unsigned phase) {
    atomicOr(&ctl->status, kStatusTimeout);
    if (atomicCAS(&ctl->diag[0], 0u, site) == 0u) {
        ctl->diag[1] = blockIdx.x | (blockIdx.y << 16);
        ctl->diag[2] = step;
        ctl->diag[3] = phase;
    }
}
static_assert(sizeof(Control) == 256, "control block is 256 bytes");

__device__ __forceinline__ unsigned ld_acquire_gpu(const unsigned* p) {
    unsigned v;
    asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_gpu(unsigned* p, unsigned v) {
    asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}

// Grid-wide barrier for a cooperative launch (all CTAs co-resident).  Thread 0
// of each CTA arrives on a counter; the last arrival resets it and releases a
// new generation.  The wait is bounded: on timeout the status word gets
// kStatusTimeout and the function returns false; the caller must then return.
__device__ __forceinline__ bool grid_barrier(Control* ctl) {
    __shared__ int s_ok;
    __syncthreads();
    if (threadIdx.x == 0) {
        int ok = 1;
        unsigned gen = ld_acquire_gpu(&ctl->bar_gen);
        __threadfence();
        unsigned arrived = atomicAdd(&ctl->bar_count, 1u);
        if (arrived == gridDim.x - 1) {
            atomicExch(&ctl->bar_count, 0u);
            __threadfence();
            st_release_gpu(&ctl->bar_gen, gen + 1);
        } else {
            const unsigned long long t0 = globaltimer_ns();
            while (ld_acquire_gpu(&ctl->bar_gen) == gen) {
                if (globaltimer_ns() - t0 > kWaitLimitNs) {
                    record_timeout(ctl, 100u, gen, 0u);
                    ok = 0;
                    break;
                }
                __nanosleep(32);
            }
        }
        __threadfence();
        s_ok = ok;
    }
    __syncthreads();
    return s_ok != 0;
}

// 8 bf16 packed in a uint4 -> 8 floats (exact).
__device__ __forceinline__ void unpack_bf16x8(const uint4& w, float* f) {
    const unsigned u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(u[i] << 16);
        f[2 * i + 1] = __uint_as_float(u[i] & 0xFFFF0000u);
    }
}

// Streaming 16-byte load through the read-only path, not kept in L1.
__device__ __forceinline__ uint4 ld_stream(const uint4* p) {
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// ---------------------------------------------------------------- formats

// Eight fp32 values -> eight E2M1 codes (round to nearest even, saturating),
// byte j = code(v[2j]) | code(v[2j+1]) << 4.
__device__ __forceinline__ uint32_t cvt_e2m1x8(const float* v) {
    uint32_t r;
    asm("{\n"
        ".reg .b8 b0, b1, b2, b3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n"
        "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n"
        "mov.b32 %0, {b0, b1, b2, b3};\n"
        "}"
        : "=r"(r)
        : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]), "f"(v[4]), "f"(v[5]), "f"(v[6]),
          "f"(v[7]));
    return r;
}

// Four bytes of E2M1 code pairs -> four f16x2 (exact).
__device__ __forceinline__ void cvt_e2m1x8_to_f16x2(uint32_t codes, uint32_t* h) {
    asm("{\n"
        ".reg .b8 b0, b1, b2, b3;\n"
        "mov.b32 {b0, b1, b2, b3}, %4;\n"
        "cvt.rn.f16x2.e2m1x2 %0, b0;\n"
        "cvt.rn.f16x2.e2m1x2 %1, b1;\n"
        "cvt.rn.f16x2.e2m1x2 %2, b2;\n"
        "cvt.rn.f16x2.e2m1x2 %3, b3;\n"
        "}"
        : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3])
        : "r"(codes));
}

// Two fp32 -> two E4M3 bytes (nearest even, saturating at 448):
// low byte from lo, high byte from hi.
__device__ __forceinline__ uint32_t cvt_e4m3x2(float lo, float hi) {
    unsigned short r;
    asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
    return r;
}

// Two E4M3 bytes (low, high) -> f16x2 (exact).
__device__ __forceinline__ uint32_t cvt_e4m3x2_to_f16x2(uint32_t two_bytes) {
    uint32_t r;
    unsigned short s = (unsigned short)two_bytes;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(r) : "h"(s));
    return r;
}

__device__ __forceinline__ float f16lo(uint32_t h2) {
    return __half2float(__ushort_as_half((unsigned short)(h2 & 0xFFFFu)));
}
__device__ __forceinline__ float f16hi(uint32_t h2) {
    return __half2float(__ushort_as_half((unsigned short)(h2 >> 16)));
}

__device__ __forceinline__ float e4m3_to_f32(uint32_t byte) {
    return f16lo(cvt_e4m3x2_to_f16x2(byte & 0xFFu));
}

// Correctly rounded x / D from r = RN(1/D): q0 = RN(x r), residual
// e = x - q0 D (exact with one fused multiply-add), q1 = RN(q0 + e r)
// (P. Markstein, "Computation of elementary functions on the IBM RISC
// System/6000 processor", IBM J. Res. Dev. 34(1), 1990).
__device__ __forceinline__ float div_markstein(float x, float D, float r) {
    float q0 = __fmul_rn(x, r);
    float e = __fmaf_rn(-q0, D, x);
    return __fmaf_rn(e, r, q0);
}

// 2^x for a pair on the FMA and integer pipes (in the attention's softmax the
// special-function unit is shared by two warps per sub-partition and is the
// scarcer resource):
// n = round(x) by adding and subtracting 1.5*2^23, f = x - n in [-1/2, 1/2],
// 2^f by a cubic (least-squares fit on relative error, max 7.5e-5), and 2^n
// added to the exponent field.  x is clamped to -125 so the result stays a
// normal number (2^f may be just below 1); the softmax's inputs are at most 8
// (the lazy-max bound), and below 2^-125 its values round to zero in fp16.
__device__ __forceinline__ float2 ex2_poly2(float2 x) {
    x.x = fmaxf(x.x, -125.0f);
    x.y = fmaxf(x.y, -125.0f);
    const float2 t = __fadd2_rn(x, make_float2(12582912.0f, 12582912.0f));
    const float2 n = __fadd2_rn(t, make_float2(-12582912.0f, -12582912.0f));
    const float2 f = __fadd2_rn(x, make_float2(-n.x, -n.y));
    float2 p = __ffma2_rn(make_float2(0.055170949548482895f, 0.055170949548482895f), f,
                          make_float2(0.2426096349954605f, 0.2426096349954605f));
    p = __ffma2_rn(p, f, make_float2(0.6932609677314758f, 0.6932609677314758f));
    p = __ffma2_rn(p, f, make_float2(0.9999281764030457f, 0.9999281764030457f));
    float2 r;
    r.x = __int_as_float(__float_as_int(p.x) + ((__float_as_int(t.x) - 0x4B400000) << 23));
    r.y = __int_as_float(__float_as_int(p.y) + ((__float_as_int(t.y) - 0x4B400000) << 23));
    return r;
}

}  // namespace nvfp4kv
