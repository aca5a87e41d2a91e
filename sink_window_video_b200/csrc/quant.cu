// quant.cu -- chunk-level NVFP4 quantization of K and V with K-smoothing and
// Four-Over-Six block scales, and the format-check kernel.
//
// Method ("2605-LongLive2" DeepRead page, Method > 推理基础设施 and
// 训练基础设施; tailorednewshub page, Inferenza W4A4 NVFP4): per chunk and per
// tensor, an FP32 tensor scale s = max|X| / (6*448); per 16-channel block an
// E4M3 scale and sixteen E2M1 codes, the block max mapped to 6 and to 4, the
// lower squared error kept; K has its per-head, per-channel mean over the
// chunk's tokens removed first and kept in fp32.
//
// One cooperative persistent kernel per chunk, four phases split by grid
// barriers.  HBM is read once (K and V, 2 bytes per element); the second
// read of each tensor hits L2 (126 MB holds both), steered by L2 eviction
// hints:
//   A. max |V|:  one streaming pass over V, per-CTA partial maxima.
//   B. the K column statistics of every (64-token segment, 256-column group)
//      -- fp32 column sums in token order, bf16 column min and max -- read
//      from HBM, and the encoding of V (its tensor scale is known after A)
//      from L2: every warp takes its statistics units first and its V units
//      after, so each SM interleaves K's HBM stream with V's arithmetic.
//   C. per column: the segment sums added in segment order and divided by
//      T (the mean); max |K - mean| from the column min/max (x -> RN(x - mean)
//      is monotone).
//   D. the encoding of K from L2.
// Encoding: two lanes per 16-element block (8 elements each, one 128-bit
// load); the block max and the two half-errors meet through one shuffle each.
// Both targets' block scales come from one paired division, their decoded
// step D and RN(1/D) from a 256-entry table per tensor, and every division
// x / D is Markstein's correctly rounded quotient (one multiply, two fused
// multiply-adds) on float pairs.
// Every fp32 step that the definition fixes is one IEEE operation (explicit
// _rn intrinsics, compiled without FMA contraction), so codes, scales, means
// and tensor scales are bit-identical to the definition.
#include "common.cuh"
#include "kernels.h"
#include "nvfp4_encode.cuh"

namespace nvfp4kv {
namespace {

constexpr int kQuantThreads = 768;       // one CTA per SM: 24 warps
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kEncTokens = 8;          // tokens per encoding unit (one warp)
constexpr int kFinCols = 32;           // columns per finalize block (one per lane)
constexpr int kFinSegs = 120;          // segments staged per finalize pass (5 per warp)
struct QuantArgs {
    const uint4* K;
    const uint4* V;
    int T, H, HD, nseg, ngroups;
    uint8_t* k_codes;
    uint8_t* k_scales;
    uint8_t* v_codes;
    uint8_t* v_scales;
    float* k_mean;
    float* tensor_scales;
    float* psum;
    uint32_t* pmin;      // bf16x2 words, [nseg][HD/2]
    uint32_t* pmax;
    float* kpart;
    float* vpart;
    Control* ctl;
    float one;              // 1 as a run-time value (see encode8_fast)
};

struct QuantShared {
    float red[kQuantWarps];
    unsigned qhead;                           // this CTA's phase-B work queue
    float2 tab[256];                          // per E4M3 code: D = RN(code * s), RN(1/D)
    uint8_t sb[kQuantWarps][kEncTokens * 8];  // staged scale bytes of one unit per warp
    float fsum[kFinSegs][kFinCols];           // finalize staging
    unsigned short fmin[kFinSegs][kFinCols];
    unsigned short fmax[kFinSegs][kFinCols];
};

__device__ __forceinline__ float block_max(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int i = 1; i < kQuantWarps; ++i) r = fmaxf(r, red[i]);
    __syncthreads();
    return r;
}

__device__ __forceinline__ __nv_bfloat162 as_bf162(uint32_t u) {
    return *reinterpret_cast<__nv_bfloat162*>(&u);
}
__device__ __forceinline__ uint32_t as_u32(__nv_bfloat162 v) {
    return *reinterpret_cast<uint32_t*>(&v);
}

// The tensor scale from the per-CTA partial maxima, and the decode table.
__device__ __forceinline__ float tensor_scale_and_table(const float* part, QuantShared& sh) {
    float m = 0.0f;
    for (int i = threadIdx.x; i < gridDim.x; i += blockDim.x) m = fmaxf(m, __ldcg(part + i));
    const float A = block_max(m, sh.red);
    const float s = A > 0.0f ? __fdiv_rn(A, kTensorScaleDiv) : 1.0f;
    for (int c = threadIdx.x; c < 256; c += blockDim.x) {
        const float D = __fmul_rn(e4m3_to_f32((uint32_t)c), s);
        sh.tab[c] = make_float2(D, D > 0.0f ? __frcp_rn(D) : 0.0f);
    }
    __syncthreads();
    return s;
}

// ---------------------------------------------------------------- phase A

__device__ void phase_vmax(const QuantArgs& a, QuantShared& sh, uint64_t keep) {
    const size_t n16 = (size_t)a.T * a.HD / 8;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t m = 0;                               // two bf16 magnitudes, lane-wise max
    for (; i + 15 * stride < n16; i += 16 * stride) {
        uint4 w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) w[k] = ld_hint(a.V + i + k * stride, keep);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            m = __vmaxu2(m, w[k].x & 0x7FFF7FFFu);
            m = __vmaxu2(m, w[k].y & 0x7FFF7FFFu);
            m = __vmaxu2(m, w[k].z & 0x7FFF7FFFu);
            m = __vmaxu2(m, w[k].w & 0x7FFF7FFFu);
        }
    }
    for (; i < n16; i += stride) {
        const uint4 w = ld_hint(a.V + i, keep);
        m = __vmaxu2(m, w.x & 0x7FFF7FFFu);
        m = __vmaxu2(m, w.y & 0x7FFF7FFFu);
        m = __vmaxu2(m, w.z & 0x7FFF7FFFu);
        m = __vmaxu2(m, w.w & 0x7FFF7FFFu);
    }
    const float v = fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
    const float b = block_max(v, sh.red);
    if (threadIdx.x == 0) {
        a.vpart[blockIdx.x] = b;
    }
}

// ---------------------------------------------------------------- K column statistics

__device__ __forceinline__ void stats_k_token(const uint4& w, float* sum, uint32_t* mn,
                                              uint32_t* mx) {
    float f[8];
    unpack_bf16x8(w, f);
#pragma unroll
    for (int i = 0; i < 8; ++i) sum[i] = __fadd_rn(sum[i], f[i]);
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        mn[j] = as_u32(__hmin2(as_bf162(mn[j]), as_bf162(u[j])));
        mx[j] = as_u32(__hmax2(as_bf162(mx[j]), as_bf162(u[j])));
    }
}

// One (64-token segment, 256-column group) of K: lane = 8 columns.
__device__ void stats_unit(const QuantArgs& a, int unit, uint64_t keep) {
    const int lane = threadIdx.x & 31;
    const int s = unit / a.ngroups;
    const int g = unit - s * a.ngroups;
    const int col = g * 256 + lane * 8;
    if (col >= a.HD) return;
    const int t0 = s * kSegment;
    const int nt = min(kSegment, a.T - t0);
    const size_t row8 = (size_t)a.HD / 8;
    const uint4* src = a.K + (size_t)t0 * row8 + col / 8;
    float sum[8];
    uint32_t mn[4], mx[4];
#pragma unroll
    for (int i = 0; i < 8; ++i) sum[i] = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) { mn[j] = 0x7F807F80u; mx[j] = 0xFF80FF80u; }
    int t = 0;
    for (; t + 16 <= nt; t += 16) {
        uint4 w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) w[k] = ld_hint(src + (size_t)(t + k) * row8, keep);
#pragma unroll
        for (int k = 0; k < 16; ++k) stats_k_token(w[k], sum, mn, mx);
    }
    for (; t < nt; ++t) stats_k_token(ld_hint(src + (size_t)t * row8, keep), sum, mn, mx);
    float4* ps = reinterpret_cast<float4*>(a.psum + (size_t)s * a.HD + col);
    ps[0] = make_float4(sum[0], sum[1], sum[2], sum[3]);
    ps[1] = make_float4(sum[4], sum[5], sum[6], sum[7]);
    const size_t w2 = ((size_t)s * a.HD + col) / 2;
    *reinterpret_cast<uint4*>(a.pmin + w2) = make_uint4(mn[0], mn[1], mn[2], mn[3]);
    *reinterpret_cast<uint4*>(a.pmax + w2) = make_uint4(mx[0], mx[1], mx[2], mx[3]);
}

// ---------------------------------------------------------------- encoding

// One unit: head h, tokens [t0, t0 + 8) of K (mean subtracted) or V (mean
// -0: x + (-0) = x exactly, signed zeros included).  Lane = (token parity,
// 8-channel group); iteration it covers tokens t0 + 2 it + {0, 1}, with the
// next iteration's 16 bytes loaded ahead.
__device__ void encode_unit(const QuantArgs& a, QuantShared& sh, bool isK, int h, int t0,
                            float s, bool fast, float ms6, float ms4, float2 rm,
                            uint64_t release) {
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int c8 = lane & 15;                 // 8-channel group of this lane
    const int tsub = lane >> 4;
    const bool odd = (lane & 1) != 0;         // second half of its 16-block
    const uint4* src = isK ? a.K : a.V;
    float2 nmu[4];
    if (isK) {
        const float4* mp = reinterpret_cast<const float4*>(a.k_mean + h * kHeadDim + c8 * 8);
        const float4 m0 = __ldcg(mp), m1 = __ldcg(mp + 1);
        nmu[0] = make_float2(-m0.x, -m0.y);
        nmu[1] = make_float2(-m0.z, -m0.w);
        nmu[2] = make_float2(-m1.x, -m1.y);
        nmu[3] = make_float2(-m1.z, -m1.w);
    } else {
#pragma unroll
        for (int j = 0; j < 4; ++j) nmu[j] = make_float2(-0.0f, -0.0f);
    }
    uint32_t* codes = reinterpret_cast<uint32_t*>(isK ? a.k_codes : a.v_codes);
    auto load = [&](int it) {
        const int t = t0 + 2 * it + tsub;
        return t < a.T ? ld_hint(src + ((size_t)t * a.H + h) * 16 + c8, release)
                       : make_uint4(0u, 0u, 0u, 0u);
    };
    uint4 wn = load(0);
#pragma unroll 1
    for (int it = 0; it < kEncTokens / 2; ++it) {
        const uint4 w = wn;
        if (it + 1 < kEncTokens / 2) wn = load(it + 1);
        const int t = t0 + 2 * it + tsub;
        float2 x[4];
        {
            const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int j = 0; j < 4; ++j) x[j] = bf16x2_add_f32x2(u[j], nmu[j]);   // RN(K - mean), or V
        }
        const float ah = max_abs8(x);
        const float ab = fmaxf(ah, __shfl_xor_sync(0xFFFFFFFFu, ah, 1));
        // block scales of both targets: RN(ab / RN(6 s)), RN(ab / RN(4 s))
        float2 rat;
        if (fast && ab >= kFastMinBlockMax) {
            const float2 AB = make_float2(ab, ab);
            const float2 q0 = __fmul2_rn(AB, rm);
            const float2 e = __ffma2_rn(q0, make_float2(-ms6, -ms4), AB);
            rat = __ffma2_rn(e, rm, q0);
        } else {
            rat = ratio_slow(ab, ms6, ms4);
        }
        const uint32_t sbp = cvt_e4m3x2(rat.x, rat.y);
        const uint32_t sb6 = sbp & 0xFFu, sb4 = sbp >> 8;
        const float2 t6 = sh.tab[sb6], t4 = sh.tab[sb4];
        uint32_t q6, q4;
        float e6, e4;
        if (fast) {
            encode8_fast(x, t6, a.one, q6, e6);
            encode8_fast(x, t4, a.one, q4, e4);
        } else {
            const Enc8 r6 = encode8_slow(x[0].x, x[0].y, x[1].x, x[1].y, x[2].x, x[2].y,
                                         x[3].x, x[3].y, t6.x);
            const Enc8 r4 = encode8_slow(x[0].x, x[0].y, x[1].x, x[1].y, x[2].x, x[2].y,
                                         x[3].x, x[3].y, t4.x);
            q6 = r6.q; e6 = r6.err;
            q4 = r4.q; e4 = r4.err;
        }
        // block error = (elements 0..7) + (elements 8..15)
        const float E6 = __fadd_rn(e6, __shfl_xor_sync(0xFFFFFFFFu, e6, 1));
        const float E4 = __fadd_rn(e4, __shfl_xor_sync(0xFFFFFFFFu, e4, 1));
        const bool keep4 = E4 < E6;
        uint32_t q = keep4 ? q4 : q6;
        if (!((keep4 ? t4.x : t6.x) > 0.0f)) q = 0u;      // a zero step stores +0 codes
        if (t < a.T) codes[((size_t)h * a.T + t) * 16 + c8] = q;
        if (!odd) sh.sb[warp][(2 * it + tsub) * 8 + (c8 >> 1)] = (uint8_t)(keep4 ? sb4 : sb6);
    }
    __syncwarp();
    if (lane < kEncTokens && t0 + lane < a.T) {
        uint8_t* scales = isK ? a.k_scales : a.v_scales;
        *reinterpret_cast<uint2*>(scales + ((size_t)h * a.T + t0 + lane) * 8) =
            *reinterpret_cast<const uint2*>(&sh.sb[warp][lane * 8]);
    }
    __syncwarp();
}

// ---------------------------------------------------------------- phase B

__device__ void phase_kstats_vencode(const QuantArgs& a, QuantShared& sh, uint64_t keep,
                                     uint64_t release) {
    if (threadIdx.x == 0) sh.qhead = 0u;
    const float sV = tensor_scale_and_table(a.vpart, sh);     // (its barriers publish qhead)
    if (blockIdx.x == 0 && threadIdx.x == 0) a.tensor_scales[1] = sV;
    const EncodeConsts c = encode_consts(sV);
    // CTA b owns an even slice of the statistics units and of the V units;
    // its warps take them from a shared-memory queue, statistics first
    // (memory-bound) and V encoding after (arithmetic), so every SM
    // interleaves K's HBM stream with V's arithmetic and no warp idles.
    const int G = gridDim.x, b = blockIdx.x;
    const int n_stats = a.nseg * a.ngroups;
    const int tiles = (a.T + kEncTokens - 1) / kEncTokens;
    const int n_v = a.H * tiles;
    const int s0 = (int)((long long)n_stats * b / G), s1 = (int)((long long)n_stats * (b + 1) / G);
    const int v0 = (int)((long long)n_v * b / G), v1 = (int)((long long)n_v * (b + 1) / G);
    const unsigned n_mine = (unsigned)((s1 - s0) + (v1 - v0));
    const int lane = threadIdx.x & 31;
    unsigned i = 0;
    if (lane == 0) i = atomicAdd(&sh.qhead, 1u);
    i = __shfl_sync(0xFFFFFFFFu, i, 0);
    while (i < n_mine) {
        unsigned next = 0;
        if (lane == 0) next = atomicAdd(&sh.qhead, 1u);
        if ((int)i < s1 - s0) {
            stats_unit(a, s0 + (int)i, keep);
        } else {
            const int u = v0 + (int)i - (s1 - s0);
            const int h = u / tiles;
            const int tile = u - h * tiles;
            encode_unit(a, sh, false, h, tile * kEncTokens, c.s, c.fast, c.ms6, c.ms4, c.rm,
                               release);
        }
        i = __shfl_sync(0xFFFFFFFFu, next, 0);
    }
}

// ---------------------------------------------------------------- phase C

__device__ void phase_finalize(const QuantArgs& a, QuantShared& sh) {
    float kp = 0.0f;
    const int nblocks = a.HD / kFinCols;
    const float Tf = (float)a.T;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const unsigned short* pmin = reinterpret_cast<const unsigned short*>(a.pmin);
    const unsigned short* pmax = reinterpret_cast<const unsigned short*>(a.pmax);
    for (int b = blockIdx.x; b < nblocks; b += gridDim.x) {
        const int col = b * kFinCols + lane;
        float S = 0.0f, mn = INFINITY, mx = -INFINITY;
        for (int s0 = 0; s0 < a.nseg; s0 += kFinSegs) {
            const int ns = min(kFinSegs, a.nseg - s0);
            // all warps stage the pass's segments, every load in flight at once ...
            float ps[kFinSegs / kQuantWarps];
            unsigned short pn[kFinSegs / kQuantWarps], px[kFinSegs / kQuantWarps];
#pragma unroll
            for (int j = 0; j < kFinSegs / kQuantWarps; ++j) {
                const int k = warp + j * kQuantWarps;
                if (k < ns) {
                    const size_t i = (size_t)(s0 + k) * a.HD + col;
                    ps[j] = __ldcg(a.psum + i);
                    pn[j] = __ldcg(pmin + i);
                    px[j] = __ldcg(pmax + i);
                }
            }
#pragma unroll
            for (int j = 0; j < kFinSegs / kQuantWarps; ++j) {
                const int k = warp + j * kQuantWarps;
                if (k < ns) {
                    sh.fsum[k][lane] = ps[j];
                    sh.fmin[k][lane] = pn[j];
                    sh.fmax[k][lane] = px[j];
                }
            }
            __syncthreads();
            // ... and warp 0 adds them in segment order
            if (warp == 0) {
                for (int k = 0; k < ns; ++k) {
                    S = __fadd_rn(S, sh.fsum[k][lane]);
                    mn = fminf(mn, __uint_as_float((uint32_t)sh.fmin[k][lane] << 16));
                    mx = fmaxf(mx, __uint_as_float((uint32_t)sh.fmax[k][lane] << 16));
                }
            }
            __syncthreads();
        }
        if (warp == 0) {
            const float mu = __fdiv_rn(S, Tf);
            a.k_mean[col] = mu;
            kp = fmaxf(kp, fmaxf(fabsf(__fsub_rn(mx, mu)), fabsf(__fsub_rn(mn, mu))));
        }
    }
    const float b = block_max(kp, sh.red);
    if (threadIdx.x == 0) a.kpart[blockIdx.x] = b;
}

// ---------------------------------------------------------------- phase D

__device__ void phase_kencode(const QuantArgs& a, QuantShared& sh, uint64_t release) {
    const float sK = tensor_scale_and_table(a.kpart, sh);
    if (blockIdx.x == 0 && threadIdx.x == 0) a.tensor_scales[0] = sK;
    const EncodeConsts c = encode_consts(sK);
    const int wg = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
    const int nw = gridDim.x * kQuantWarps;
    const int tiles = (a.T + kEncTokens - 1) / kEncTokens;
    for (int u = wg; u < a.H * tiles; u += nw) {
        const int h = u / tiles;
        const int tile = u - h * tiles;
        encode_unit(a, sh, true, h, tile * kEncTokens, c.s, c.fast, c.ms6, c.ms4, c.rm, release);
    }
}

// CTA 0 records when it starts, when it finishes its share of each phase and
// when it leaves each grid barrier (then the last CTA has arrived): a
// per-phase profile of the launch.
__device__ __forceinline__ void stamp(const QuantArgs& a, int i) {
    if (blockIdx.x == 0 && threadIdx.x == 0) a.ctl->stamp[i] = globaltimer_ns();
}

__global__ void __launch_bounds__(kQuantThreads, 1) quantize_kernel(QuantArgs a) {
    __shared__ QuantShared sh;
    const uint64_t keep = policy_keep(), release = policy_release();
    stamp(a, 0);
    phase_vmax(a, sh, keep);
    stamp(a, 1);
    if (!grid_barrier(a.ctl)) return;
    stamp(a, 2);
    phase_kstats_vencode(a, sh, keep, release);
    stamp(a, 3);
    if (!grid_barrier(a.ctl)) return;
    stamp(a, 4);
    phase_finalize(a, sh);
    stamp(a, 5);
    if (!grid_barrier(a.ctl)) return;
    stamp(a, 6);
    phase_kencode(a, sh, release);
    stamp(a, 7);
}

// ---------------------------------------------------------------- sequence-parallel phases
//
// The quantizer split at its global reductions, for a chunk whose tokens are
// spread over several GPUs (one contiguous, 64-token-aligned shard each):
//   stats:    per shard, the K column statistics of its 64-token segments and
//             its max |V| (atomicMax on the float's bits: non-negative floats
//             order like their bit patterns);
//   (the caller gathers every shard's segment statistics in token order and
//    takes the maximum of the max |V| values)
//   finalize: the mean and max |K - mean| per column from all segments, in
//             segment order -- the same fp32 sequence as the one-GPU kernel;
//   scales:   the two tensor scales;
//   encode:   per shard, the encoding of its tokens with the chunk's mean and
//             tensor scales.
// Each is an ordinary launch (no grid barrier); the results equal the one-GPU
// quantization bit for bit.

__global__ void __launch_bounds__(kQuantThreads, 1) sp_stats_kernel(QuantArgs a,
                                                                      unsigned* vmax_bits) {
    __shared__ QuantShared sh;
    const uint64_t keep = policy_keep();
    const int wg = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
    const int nw = gridDim.x * kQuantWarps;
    for (int u = wg; u < a.nseg * a.ngroups; u += nw) stats_unit(a, u, keep);
    phase_vmax(a, sh, keep);                 // per-CTA max |V| into vpart[blockIdx.x] ...
    if (threadIdx.x == 0) atomicMax(vmax_bits, __float_as_uint(a.vpart[blockIdx.x]));
}

__global__ void __launch_bounds__(kQuantThreads, 1) sp_finalize_kernel(QuantArgs a) {
    __shared__ QuantShared sh;
    phase_finalize(a, sh);                   // k_mean, per-CTA max |K - mean| in kpart
}

// max over the per-CTA partial maxima of |K - mean| and the given max |V|:
// the two amaxes (amax_out, when given) and the tensor scales s = amax / 2688
// (1 for an all-zero tensor; tensor_scales, when given).
__global__ void sp_scales_kernel(const float* kpart, int n_part, const float* vmax,
                                 float* amax_out, float* tensor_scales) {
    __shared__ float red[32];
    float m = 0.0f;
    for (int i = threadIdx.x; i < n_part; i += blockDim.x) m = fmaxf(m, kpart[i]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x == 0) {
        float A = 0.0f;
        for (int i = 0; i < (int)(blockDim.x >> 5); ++i) A = fmaxf(A, red[i]);
        const float V = *vmax;
        if (amax_out) {
            amax_out[0] = A;
            amax_out[1] = V;
        }
        if (tensor_scales) {
            tensor_scales[0] = A > 0.0f ? __fdiv_rn(A, kTensorScaleDiv) : 1.0f;
            tensor_scales[1] = V > 0.0f ? __fdiv_rn(V, kTensorScaleDiv) : 1.0f;
        }
    }
}

// blockIdx.y: 0 encodes V, 1 encodes K.
__global__ void __launch_bounds__(kQuantThreads, 1) sp_encode_kernel(QuantArgs a) {
    __shared__ QuantShared sh;
    const bool isK = blockIdx.y == 1;
    const float st = a.tensor_scales[isK ? 0 : 1];
    for (int c = threadIdx.x; c < 256; c += blockDim.x) {
        const float D = __fmul_rn(e4m3_to_f32((uint32_t)c), st);
        sh.tab[c] = make_float2(D, D > 0.0f ? __frcp_rn(D) : 0.0f);
    }
    __syncthreads();
    const EncodeConsts c = encode_consts(st);
    const uint64_t release = policy_release();
    const int wg = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
    const int nw = gridDim.x * kQuantWarps;
    const int tiles = (a.T + kEncTokens - 1) / kEncTokens;
    for (int u = wg; u < a.H * tiles; u += nw) {
        const int h = u / tiles;
        const int tile = u - h * tiles;
        encode_unit(a, sh, isK, h, tile * kEncTokens, c.s, c.fast, c.ms6, c.ms4, c.rm, release);
    }
}

// ---------------------------------------------------------------- format checks

__global__ void check_formats_kernel(int op, const float* fin, const uint8_t* bin, uint8_t* bout,
                                     float* fout, size_t n) {
    const size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    if (i >= n) return;
    switch (op) {
        case 0: {   // fp32 -> E2M1 code (low nibble of the pair with a zero partner)
            float v[8] = {fin[i], 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
            bout[i] = (uint8_t)(cvt_e2m1x8(v) & 0xFu);
            break;
        }
        case 1:
            bout[i] = (uint8_t)(cvt_e4m3x2(fin[i], 0.0f) & 0xFFu);
            break;
        case 2: {
            uint32_t h[4];
            cvt_e2m1x8_to_f16x2((uint32_t)(bin[i] & 0xFu), h);
            fout[i] = f16lo(h[0]);
            break;
        }
        case 3:
            fout[i] = e4m3_to_f32(bin[i]);
            break;
        case 4: {
            const float x = fin[2 * i], D = fin[2 * i + 1];
            fout[i] = div_markstein(x, D, __frcp_rn(D));
            break;
        }
        case 5:
            fout[i] = ex2_poly2(make_float2(fin[i], fin[i])).x;
            break;
        default:
            break;
    }
}

int g_quant_grid[64];   // cooperative grid size per device ordinal (0 = not yet known)

}  // namespace

nvfp4kv_status launch_quantize(const void* K, const void* V, int T, int H,
                               const nvfp4kv_chunk_view& out, void* ws, cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4KV_ERR_CUDA;
    if (g_quant_grid[dev] == 0) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4KV_ERR_CUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, quantize_kernel, kQuantThreads,
                                                          0) != cudaSuccess || per_sm < 1)
            return NVFP4KV_ERR_CUDA;
        g_quant_grid[dev] = min(sms * per_sm, kMaxGrid);
    }
    const WsLayout L = ws_layout(T, H);
    char* w = static_cast<char*>(ws);
    QuantArgs a;
    a.K = static_cast<const uint4*>(K);
    a.V = static_cast<const uint4*>(V);
    a.T = T;
    a.H = H;
    a.HD = H * kHeadDim;
    a.nseg = (T + kSegment - 1) / kSegment;
    a.ngroups = (a.HD + 255) / 256;
    a.k_codes = out.k_codes;
    a.k_scales = out.k_scales;
    a.v_codes = out.v_codes;
    a.v_scales = out.v_scales;
    a.k_mean = out.k_mean;
    a.tensor_scales = out.tensor_scales;
    a.psum = reinterpret_cast<float*>(w + L.psum);
    a.pmin = reinterpret_cast<uint32_t*>(w + L.pmin);
    a.pmax = reinterpret_cast<uint32_t*>(w + L.pmax);
    a.kpart = reinterpret_cast<float*>(w + L.kpart);
    a.vpart = reinterpret_cast<float*>(w + L.vpart);
    a.ctl = reinterpret_cast<Control*>(w);
    a.one = 1.0f;
    void* args[] = {&a};
    cudaError_t e = cudaLaunchCooperativeKernel((const void*)quantize_kernel,
                                                dim3(g_quant_grid[dev]), dim3(kQuantThreads),
                                                args, 0, stream);
    return e == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

nvfp4kv_status launch_check_formats(int op, const void* in, void* out, size_t n,
                                    cudaStream_t stream) {
    if (n == 0) return NVFP4KV_OK;
    const int threads = 256;
    const unsigned blocks = (unsigned)((n + threads - 1) / threads);
    check_formats_kernel<<<blocks, threads, 0, stream>>>(
        op, static_cast<const float*>(in), static_cast<const uint8_t*>(in),
        static_cast<uint8_t*>(out), static_cast<float*>(out), n);
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

int sm_count_cached() {
    static int sms[64];
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
    if (sms[dev] == 0 &&
        cudaDeviceGetAttribute(&sms[dev], cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        sms[dev] = 0;
    return sms[dev];
}

nvfp4kv_status launch_sp_stats(const void* K, const void* V, int T_local, int H, float* psum,
                               void* pmin, void* pmax, float* vmax, void* ws,
                               cudaStream_t stream) {
    const int G = sm_count_cached();
    if (G <= 0) return NVFP4KV_ERR_CUDA;
    const WsLayout L = ws_layout(T_local, H);
    QuantArgs a = {};
    a.K = static_cast<const uint4*>(K);
    a.V = static_cast<const uint4*>(V);
    a.T = T_local;
    a.H = H;
    a.HD = H * kHeadDim;
    a.nseg = (T_local + kSegment - 1) / kSegment;
    a.ngroups = (a.HD + 255) / 256;
    a.psum = psum;
    a.pmin = static_cast<uint32_t*>(pmin);
    a.pmax = static_cast<uint32_t*>(pmax);
    a.vpart = reinterpret_cast<float*>(static_cast<char*>(ws) + L.vpart);
    a.one = 1.0f;
    if (cudaMemsetAsync(vmax, 0, sizeof(float), stream) != cudaSuccess) return NVFP4KV_ERR_CUDA;
    sp_stats_kernel<<<G, kQuantThreads, 0, stream>>>(a, reinterpret_cast<unsigned*>(vmax));
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

nvfp4kv_status launch_sp_finalize(const float* psum, const void* pmin, const void* pmax,
                                  int nseg, int T, int H, const float* vmax, float* k_mean,
                                  float* amax, float* tensor_scales, void* ws,
                                  cudaStream_t stream) {
    const int HD = H * kHeadDim;
    const int nblocks = HD / kFinCols;
    const int G = min(nblocks, kMaxGrid);
    QuantArgs a = {};
    a.T = T;
    a.H = H;
    a.HD = HD;
    a.nseg = nseg;
    a.psum = const_cast<float*>(psum);
    a.pmin = static_cast<uint32_t*>(const_cast<void*>(pmin));
    a.pmax = static_cast<uint32_t*>(const_cast<void*>(pmax));
    a.k_mean = k_mean;
    a.kpart = reinterpret_cast<float*>(static_cast<char*>(ws) + ws_layout(1, H).kpart);
    sp_finalize_kernel<<<G, kQuantThreads, 0, stream>>>(a);
    if (cudaGetLastError() != cudaSuccess) return NVFP4KV_ERR_CUDA;
    sp_scales_kernel<<<1, 1024, 0, stream>>>(a.kpart, G, vmax, amax, tensor_scales);
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

nvfp4kv_status launch_scales_from_amax(const float* amax, float* tensor_scales,
                                       cudaStream_t stream) {
    sp_scales_kernel<<<1, 32, 0, stream>>>(amax, 1, amax + 1, nullptr, tensor_scales);
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

nvfp4kv_status launch_sp_encode(const void* K, const void* V, int T_local, int H,
                                const float* k_mean, const float* tensor_scales,
                                const nvfp4kv_chunk_view& out, cudaStream_t stream) {
    const int G = sm_count_cached();
    if (G <= 0) return NVFP4KV_ERR_CUDA;
    QuantArgs a = {};
    a.K = static_cast<const uint4*>(K);
    a.V = static_cast<const uint4*>(V);
    a.T = T_local;
    a.H = H;
    a.HD = H * kHeadDim;
    a.k_codes = out.k_codes;
    a.k_scales = out.k_scales;
    a.v_codes = out.v_codes;
    a.v_scales = out.v_scales;
    a.k_mean = const_cast<float*>(k_mean);
    a.tensor_scales = const_cast<float*>(tensor_scales);
    a.one = 1.0f;
    sp_encode_kernel<<<dim3((G + 1) / 2, 2), kQuantThreads, 0, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

}  // namespace nvfp4kv

// ---------------------------------------------------------------- no-allocation entry point
//
// The same quantization for callers that cannot allocate device memory: the
// scratch lives in one array compiled into the library.  Host code only sees
// a stand-in for that array's name; its device address comes from
// cudaGetSymbolAddress, taken once per device with that device current.
#include <mutex>

namespace nvfp4kv {

constexpr size_t kStaticScratchBytes = size_t(4) << 20;    // 4 MiB per GPU

static __device__ __align__(256) unsigned char g_quant_scratch[kStaticScratchBytes];

namespace {
std::mutex g_scratch_mutex;
void* g_scratch_addr[64];       // device address of g_quant_scratch, per device ordinal
}  // namespace

}  // namespace nvfp4kv

extern "C" nvfp4kv_status nvfp4kv_quantize_chunk_noalloc(const void* K, const void* V, int T_c,
                                                         int H, int d,
                                                         const nvfp4kv_chunk_view* out,
                                                         nvfp4kv_stream_t stream) {
    using namespace nvfp4kv;
    // the workspace entry point's checks, in its order
    const nvfp4kv_status st = check_quantize_chunk_args(K, V, T_c, H, d, out, nullptr, false);
    if (st != NVFP4KV_OK) return st;
    // the chunk's scratch must fit the compiled-in array
    if (ws_layout(T_c, H).quant_total > kStaticScratchBytes) return NVFP4KV_ERR_CAPACITY;

    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4KV_ERR_CUDA;
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lock(g_scratch_mutex);
        if (g_scratch_addr[dev] == nullptr) {
            void* p = nullptr;
            if (cudaGetSymbolAddress(&p, g_quant_scratch) != cudaSuccess || p == nullptr)
                return NVFP4KV_ERR_CUDA;
            g_scratch_addr[dev] = p;
        }
        scratch = g_scratch_addr[dev];
    }
    // the grid barrier and the status word must start at zero; the partial
    // sums and maxima are written before they are read
    nvfp4kv_status r = NVFP4KV_ERR_CUDA;
    if (cudaMemsetAsync(scratch, 0, sizeof(Control), (cudaStream_t)stream) == cudaSuccess)
        r = launch_quantize(K, V, T_c, H, *out, scratch, (cudaStream_t)stream);
    if (r == NVFP4KV_ERR_CUDA) {
        // the cached address may be stale (a context that was reset and
        // recreated reloads the module): look it up again on the next call
        std::lock_guard<std::mutex> lock(g_scratch_mutex);
        g_scratch_addr[dev] = nullptr;
    }
    return r;
}
