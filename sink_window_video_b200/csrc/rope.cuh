// rope.cuh -- device helpers of the 3D rotary position embedding (rope.cu and
// the chunk quantizer's fused K path in quant.cu).
//
// Table of a chunk in device memory, float2 entries {cos, sin} (fp32):
//   [0, frames*22)                      frame part: entry f*22 + i, the frame
//                                       coordinate frame_pos0 + f, pair i of 22;
//   [frames*22, + rows*21)              row part: entry r*21 + i, pair i of 21;
//   [frames*22 + rows*21, + cols*21)    column part: entry c*21 + i.
// Head channels (d = 128): frame pairs 0..21 (channels 0..43), row pairs
// 22..42 (44..85), column pairs 43..63 (86..127).
//
// The chunk quantizer stages the table in shared memory, one row per
// coordinate with head pair P at slot P + P/4 (less the part's first slot):
// lanes that take head pairs 4 apart then read different banks, and the four
// pairs of an aligned group P0..P0+3 sit in consecutive slots.  rope_kernel
// reads its few entries per token straight from the device table.
#pragma once

#include <cuda_bf16.h>
#include <cstdint>

#include "kernels.h"

namespace nvfp4kv {

constexpr int kRopeFramePairs = 22;       // 44 channels
constexpr int kRopeAxisPairs = 21;        // 42 channels each for rows and columns
constexpr int kRopeRowPair0 = kRopeFramePairs;                    // first row pair
constexpr int kRopeColPair0 = kRopeFramePairs + kRopeAxisPairs;   // first column pair

__host__ __device__ constexpr int rope_pslot(int P) { return P + (P >> 2); }
constexpr int kRopeFrameRow = rope_pslot(kRopeRowPair0 - 1) + 1;                    // 27
constexpr int kRopeRowRow = rope_pslot(kRopeColPair0 - 1) - rope_pslot(kRopeRowPair0) + 1;  // 26
constexpr int kRopeColRow = rope_pslot(63) - rope_pslot(kRopeColPair0) + 1;          // 26

__host__ __device__ inline int rope_staged_slots(int frames, int rows, int cols) {
    return frames * kRopeFrameRow + rows * kRopeRowRow + cols * kRopeColRow;
}

// Token geometry of a rotation: the table and the frame grid, with the
// reciprocals m = floor(2^32 / D) + 1 of rows*cols and cols, so that
// t / D = umulhi(t, m) exactly whenever t * D < 2^32: m D - 2^32 = e lies in
// (0, D], and t e < 2^32 keeps the fraction below 1.  D = 1 (m = 2^32 does
// not fit) is marked by m = 0 and divides as t itself.
struct RopeDev {
    const float2* tab;             // device table (entries above)
    int frames, rows, cols, rc;
    int entries;                   // frames*22 + (rows + cols)*21
    int rowslot, colslot;          // first staged slot of the row and column parts
    uint32_t m_rc, m_c;
    float one;                     // 1 as a run-time value (see rope_pair)
};

// The device view of a rotation's geometry (rope.cu).
RopeDev rope_dev(const RopeGeom& r);

__host__ __device__ inline uint32_t rope_reciprocal(uint32_t D) {
    return D > 1 ? (uint32_t)((1ull << 32) / D + 1ull) : 0u;
}

__device__ __forceinline__ uint32_t rope_div(uint32_t t, uint32_t m) {
    return m ? __umulhi(t, m) : t;
}

// Copy the table into shared memory sm (rope_staged_slots float2), every
// thread of the CTA taking a share; the caller synchronizes the CTA.
__device__ __forceinline__ void rope_stage(const RopeDev& g, float2* sm) {
    const int nf = g.frames * kRopeFramePairs;
    const int nr = g.rows * kRopeAxisPairs;
    for (int e = threadIdx.x; e < g.entries; e += blockDim.x) {
        int slot;
        if (e < nf) {
            const int f = e / kRopeFramePairs, P = e - f * kRopeFramePairs;
            slot = f * kRopeFrameRow + rope_pslot(P);
        } else if (e < nf + nr) {
            const int k = e - nf, r = k / kRopeAxisPairs;
            const int P = kRopeRowPair0 + k - r * kRopeAxisPairs;
            slot = g.rowslot + r * kRopeRowRow + rope_pslot(P) - rope_pslot(kRopeRowPair0);
        } else {
            const int k = e - nf - nr, c = k / kRopeAxisPairs;
            const int P = kRopeColPair0 + k - c * kRopeAxisPairs;
            slot = g.colslot + c * kRopeColRow + rope_pslot(P) - rope_pslot(kRopeColPair0);
        }
        sm[slot] = __ldg(g.tab + e);
    }
}

// The staged slots of an aligned group of four head pairs P0..P0+3 (P0 % 4 ==
// 0) for one token: pair j is at slot (j < split ? a : b) + j.  A group lies in
// one part except [20, 23] (frame, row: split 2) and [40, 43] (row, column:
// split 3).
struct RopeGroup {
    int P0, split;
    int partA, partB;               // 0 frame, 1 row, 2 column
};

__device__ __forceinline__ int rope_part(int P) {
    return P < kRopeRowPair0 ? 0 : (P < kRopeColPair0 ? 1 : 2);
}

__device__ __forceinline__ RopeGroup rope_group(int P0) {
    RopeGroup q;
    q.P0 = P0;
    q.partA = rope_part(P0);
    q.partB = rope_part(P0 + 3);
    q.split = q.partA == q.partB ? 4 : (q.partA == 0 ? kRopeRowPair0 - P0 : kRopeColPair0 - P0);
    return q;
}

// Slot bases of token t's three rows: slot of head pair P = base[part] + pslot(P).
struct RopeRows {
    int f, r, c;
};

__device__ __forceinline__ RopeRows rope_rows(const RopeDev& g, uint32_t t) {
    const uint32_t f = rope_div(t, g.m_rc);
    const uint32_t rem = t - f * (uint32_t)g.rc;
    const uint32_t r = rope_div(rem, g.m_c);
    const uint32_t c = rem - r * (uint32_t)g.cols;
    RopeRows b;
    b.f = (int)f * kRopeFrameRow;
    b.r = g.rowslot + (int)r * kRopeRowRow - rope_pslot(kRopeRowPair0);
    b.c = g.colslot + (int)c * kRopeColRow - rope_pslot(kRopeColPair0);
    return b;
}

__device__ __forceinline__ int rope_row_of(const RopeRows& b, int part) {
    return part == 0 ? b.f : (part == 1 ? b.r : b.c);
}

// One bf16 channel pair u = (x0 low half, x1 high half) turned by the entry
// {cos, sin}: (x0 cos - x1 sin, x1 cos + x0 sin), one fp32 rounding per
// product and per sum, each result rounded to bf16 (RN-even).  The sums are
// fma(product, -+one, product) with `one` a run-time 1 (p * -1 and p * 1 are
// exact): a separate multiply and add may be fused by the compiler into one
// fma, which skips the rounding of a product (and moves results that sit on a
// bf16 tie); a multiply cannot be merged into the multiplicand of an fma.
__device__ __forceinline__ uint32_t rope_pair(uint32_t u, float2 cs, float one) {
    const float2 x = make_float2(__uint_as_float(u << 16), __uint_as_float(u & 0xFFFF0000u));
    const float2 a = __fmul2_rn(x, make_float2(cs.x, cs.x));      // x0 cos, x1 cos
    const float2 b = __fmul2_rn(x, make_float2(cs.y, cs.y));      // x0 sin, x1 sin
    const float y0 = __fmaf_rn(b.y, -one, a.x);
    const float y1 = __fmaf_rn(b.x, one, a.y);
    const __nv_bfloat162 r = __floats2bfloat162_rn(y0, y1);
    return *reinterpret_cast<const uint32_t*>(&r);
}

// The four channel pairs of group q (words u[0..3]) of token rows b, turned
// with the staged table sm.
__device__ __forceinline__ void rope_group4(const RopeGroup& q, const RopeRows& b,
                                            const float2* sm, float one, uint32_t* u) {
    const int base = rope_pslot(q.P0);
    const int sa = rope_row_of(b, q.partA) + base;
    const int sb = rope_row_of(b, q.partB) + base;
#pragma unroll
    for (int j = 0; j < 4; ++j) u[j] = rope_pair(u[j], sm[(j < q.split ? sa : sb) + j], one);
}

}  // namespace nvfp4kv
