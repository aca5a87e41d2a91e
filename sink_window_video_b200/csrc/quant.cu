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
// One cooperative persistent kernel per chunk (one CTA of 24 warps per SM).
// HBM is read once (K and V, 2 bytes per element); the encoding re-reads each
// tensor from L2 (126 MB holds both), steered by L2 eviction hints.  The CTAs
// never wait at a grid-wide barrier: they publish their progress in counters
// of the workspace's control block, and a warp waits (bounded in time) only
// for the one result it needs next:
//   1. all warps: max |V| over an even slice of V (read from HBM, kept in
//      L2); each CTA folds its maximum into a global atomic maximum and counts
//      itself in.
//   2. warps 0-9 ("statistics warps"): the K column statistics of the CTA's
//      (64-token segment, 256-column group) units -- fp32 column sums in
//      token order, bf16 column minima and maxima -- read from HBM; then, once
//      every CTA's statistics are in, the mean of the CTA's 32-column blocks
//      (segment sums added in segment order, / T) and max |K - mean| per
//      column from its minimum and maximum (x -> RN(x - mean) is monotone),
//      folded into a global atomic maximum.
//      warps 10-23, and the statistics warps after that: the encoding of V
//      (its tensor scale is known once every CTA has counted in), so K's HBM
//      stream overlaps V's arithmetic on every SM.
//   3. all warps: the encoding of K, once every column block is finalized.
// The last CTA to finish resets the counters for the next launch.
// Encoding: one lane per 16-element block (two 128-bit loads), four tokens of
// a head per warp and step, see encode_block16 (nvfp4_encode.cuh): both
// targets' scales from one paired division, codes of correctly rounded
// quotients, the candidates compared on error estimates with the definition's
// exact sums whenever the estimates are close.
// Every fp32 step that the definition fixes is one IEEE operation (explicit
// _rn intrinsics, compiled without FMA contraction), so codes, scales, means
// and tensor scales are bit-identical to the definition.
#include <cstddef>

#include "common.cuh"
#include "kernels.h"
#include "nvfp4_encode.cuh"
#include "rope.cuh"

namespace nvfp4kv {
namespace {

constexpr int kQuantThreads = 768;       // one CTA per SM: 24 warps
constexpr int kQuantWarps = kQuantThreads / 32;
constexpr int kStatsWarps = 10;          // warps 0-9 read K's statistics first
constexpr int kStatsWarpsRope = 15;      // with K rotated: its statistics cost ~3x
constexpr int kEncTokens = 16;           // tokens per encoding unit (one warp)
constexpr int kFinCols = 32;             // columns per finalize block (one per lane)
constexpr int kStatsBatch = 8;           // K rows in flight per lane in the statistics pass
constexpr int kFinSegs = 120;            // segments staged per finalize pass
static_assert(kFinSegs % kStatsWarps == 0 && kFinSegs % kStatsWarpsRope == 0,
              "finalize staging splits evenly");

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
    RopeDev rope;           // quantize_kernel<true>: K is rotated first (rope.cu)
};

// Shared memory of the chunk quantizer (the sequence-parallel kernels use the
// table and the staging areas).
struct QuantShared {
    float red[kQuantWarps];
    float2 tab[2][256];                       // per E4M3 code: D = RN(code * s), RN(1/D); [V, K]
    float s[2];                               // tensor scales [V, K]
    int ready[2];                             // tables built (1) or given up (-1)
    int claim[2];                             // table builder election
    int abort;                                // a wait of this CTA gave up
    int fin_go;                               // the statistics warps may finalize
    unsigned q_stats, q_v, q_k;               // this CTA's work queues
    alignas(16) uint8_t sb[kQuantWarps][kEncTokens * 8];  // staged scale bytes of a unit per warp
    float fsum[kFinSegs][kFinCols];           // finalize staging
    unsigned short fmin[kFinSegs][kFinCols];
    unsigned short fmax[kFinSegs][kFinCols];
};
// a staged row of 8 scale bytes is copied out as one 8-byte word
static_assert(offsetof(QuantShared, sb) % 16 == 0, "scale staging is 16-byte aligned");

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

// The decode table of one tensor: per E4M3 code c, D = RN(decode(c) * s) and
// RN(1/D) (0 for D = 0), entries [first, 256) in steps of `step`.
__device__ __forceinline__ void fill_table(float2* tab, float s, int first, int step) {
    for (int c = first; c < 256; c += step) {
        const float D = __fmul_rn(e4m3_to_f32((uint32_t)c), s);
        tab[c] = make_float2(D, D > 0.0f ? __frcp_rn(D) : 0.0f);
    }
}

// ---------------------------------------------------------------- bounded waits

// Wait (one thread) until *counter == target; gives up at the time limit, or
// at once when this CTA already gave up somewhere.
__device__ bool wait_counter(const unsigned* counter, unsigned target, Control* ctl,
                             volatile int* abort, unsigned site) {
    const unsigned long long t0 = globaltimer_ns();
    while (ld_acquire_gpu(counter) != target) {
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            record_timeout(ctl, site, target, 0u);
            *abort = 1;
            return false;
        }
        __nanosleep(64);
    }
    return true;
}

// The tensor scale and decode table of V (which = 0) or K (1) in this CTA's
// shared memory.  The first warp to ask builds it, once the global maximum is
// complete (every CTA counted in, resp. every column block finalized); the
// others wait for it.  Returns false when a wait gave up.
__device__ bool ensure_table(const QuantArgs& a, QuantShared& sh, int which) {
    volatile int* ready = &sh.ready[which];
    const int lane = threadIdx.x & 31;
    int state = *ready;
    if (state == 0) {
        int mine = 0;
        if (lane == 0) mine = atomicCAS(&sh.claim[which], 0, 1) == 0;
        mine = __shfl_sync(0xFFFFFFFFu, mine, 0);
        if (mine) {
            int ok = 1;
            if (lane == 0) {
                ok = which == 0 ? wait_counter(&a.ctl->q_vdone, gridDim.x, a.ctl, &sh.abort, 101u)
                                : wait_counter(&a.ctl->q_fdone, (unsigned)(a.HD / kFinCols),
                                               a.ctl, &sh.abort, 102u);
            }
            ok = __shfl_sync(0xFFFFFFFFu, ok, 0);
            if (!ok) {
                if (lane == 0) *ready = -1;
                return false;
            }
            const float A = __uint_as_float(ld_acquire_gpu(which == 0 ? &a.ctl->q_vmax
                                                                      : &a.ctl->q_kmax));
            const float s = A > 0.0f ? __fdiv_rn(A, kTensorScaleDiv) : 1.0f;
            fill_table(sh.tab[which], s, lane, 32);
            if (lane == 0) {
                sh.s[which] = s;
                if (blockIdx.x == 0) a.tensor_scales[which == 0 ? 1 : 0] = s;
            }
            __threadfence_block();
            __syncwarp();
            if (lane == 0) *ready = 1;
            return true;
        }
        if (lane == 0) {
            // twice the builder's limit: a builder that gives up is the wait recorded
            const unsigned long long t0 = globaltimer_ns();
            while ((state = *ready) == 0) {
                if (sh.abort) break;
                if (globaltimer_ns() - t0 > 2 * kWaitLimitNs) {
                    record_timeout(a.ctl, 103u + which, 0u, 0u);
                    sh.abort = 1;
                    break;
                }
                __nanosleep(64);
            }
        }
        state = __shfl_sync(0xFFFFFFFFu, *ready, 0);
    }
    __threadfence_block();
    return state == 1;
}

// ---------------------------------------------------------------- max |V|

// max |V| over this CTA's even slice (all threads of the CTA), one streaming
// pass; the CTA's maximum goes to vpart[blockIdx.x] and is returned.
__device__ float phase_vmax(const QuantArgs& a, QuantShared& sh, uint64_t keep) {
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
    if (threadIdx.x == 0) a.vpart[blockIdx.x] = b;
    return b;
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

// K rotated (rope.cu's reading): the 8 channels of w, head pair group q, of
// token t, with the table staged in shared memory (rsm).
__device__ __forceinline__ uint4 rope_k8(const RopeDev& g, const float2* rsm, const RopeGroup& q,
                                         uint4 w, int t) {
    uint32_t u[4] = {w.x, w.y, w.z, w.w};
    rope_group4(q, rope_rows(g, (uint32_t)t), rsm, g.one, u);
    return make_uint4(u[0], u[1], u[2], u[3]);
}

// One (64-token segment, 256-column group) of K: lane = 8 columns (with ROPE,
// of the rotated K).
template <bool ROPE>
__device__ void stats_unit(const QuantArgs& a, const float2* rsm, int unit, uint64_t keep) {
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
    const RopeGroup grp = rope_group((lane & 15) * 4);   // the lane's four head pairs
    int t = 0;
    for (; t + kStatsBatch <= nt; t += kStatsBatch) {
        uint4 w[kStatsBatch];
#pragma unroll
        for (int k = 0; k < kStatsBatch; ++k) w[k] = ld_hint(src + (size_t)(t + k) * row8, keep);
#pragma unroll
        for (int k = 0; k < kStatsBatch; ++k) {
            if (ROPE) w[k] = rope_k8(a.rope, rsm, grp, w[k], t0 + t + k);
            stats_k_token(w[k], sum, mn, mx);
        }
    }
    for (; t < nt; ++t) {
        uint4 w = ld_hint(src + (size_t)t * row8, keep);
        if (ROPE) w = rope_k8(a.rope, rsm, grp, w, t0 + t);
        stats_k_token(w, sum, mn, mx);
    }
    float4* ps = reinterpret_cast<float4*>(a.psum + (size_t)s * a.HD + col);
    ps[0] = make_float4(sum[0], sum[1], sum[2], sum[3]);
    ps[1] = make_float4(sum[4], sum[5], sum[6], sum[7]);
    const size_t w2 = ((size_t)s * a.HD + col) / 2;
    *reinterpret_cast<uint4*>(a.pmin + w2) = make_uint4(mn[0], mn[1], mn[2], mn[3]);
    *reinterpret_cast<uint4*>(a.pmax + w2) = make_uint4(mx[0], mx[1], mx[2], mx[3]);
}

// ---------------------------------------------------------------- encoding

// One unit: head h, tokens [t0, t0 + kEncTokens) of K (mean subtracted) or V
// (mean -0: x + (-0) = x exactly, signed zeros included).  Lane = (token
// within a step, 16-channel block), one block per lane (encode_block16);
// step it covers tokens t0 + 4 it + {0..3}, with the next step's loads in
// flight.
template <bool IS_K, bool ROPE>
__device__ void encode_unit(const QuantArgs& a, const float2* tab, const EncodeConsts& c,
                            uint8_t* sbst, int h, int t0, uint64_t release,
                            const float2* rsm = nullptr) {
    const int lane = threadIdx.x & 31;
    const int blk = lane & 7;                 // 16-channel block of this lane
    const int tsub = lane >> 3;               // token within a step
    // K: this lane's 16 channel means, re-read from L1 every step (held in
    // registers they would push the encoder out of them)
    const float4* mp = reinterpret_cast<const float4*>(a.k_mean + h * kHeadDim + blk * 16);
    const size_t row4 = (size_t)a.H * 64;                       // uint4 per four tokens
    const uint4* src = (IS_K ? a.K : a.V) + ((size_t)(t0 + tsub) * a.H + h) * 16 + blk * 2;
    uint2* dst = reinterpret_cast<uint2*>(IS_K ? a.k_codes : a.v_codes) +
                 ((size_t)h * a.T + t0 + tsub) * 8 + blk;
    uint8_t* sbw = sbst + tsub * 8 + blk;
    constexpr int kIters = kEncTokens / 4;
    // a whole unit needs no per-token check; a ragged last unit reads and
    // writes only its tokens (zeros stand in for the rest)
    const bool full = t0 + kEncTokens <= a.T;
    const int nt = a.T - t0 - tsub;
    auto load = [&](int it, const uint4* p, uint4& w0, uint4& w1) {
        if (full || 4 * it < nt) {
            w0 = ld_hint(p, release);
            w1 = ld_hint(p + 1, release);
        } else {
            w0 = w1 = make_uint4(0u, 0u, 0u, 0u);
        }
    };
    uint4 a0, a1;
    load(0, src, a0, a1);
    const uint4* pf = src + row4;
#pragma unroll 1
    for (int it = 0; it < kIters; ++it) {
        const uint4 w0 = a0, w1 = a1;
        if (it + 1 < kIters) {
            load(it + 1, pf, a0, a1);
            pf += row4;
        }
        float2 x[8];
        {
            uint32_t u[8] = {w0.x, w0.y, w0.z, w0.w, w1.x, w1.y, w1.z, w1.w};
            if (IS_K && ROPE && (full || 4 * it < nt)) {
                // the rotated K: head pairs 8 blk .. 8 blk + 7 of this lane's token
                const RopeRows b = rope_rows(a.rope, (uint32_t)(t0 + tsub + 4 * it));
                rope_group4(rope_group(8 * blk), b, rsm, a.rope.one, u);
                rope_group4(rope_group(8 * blk + 4), b, rsm, a.rope.one, u + 4);
            }
#pragma unroll
            for (int j = 0; j < 8; ++j)
                // bf16 -> fp32 exactly (signed zeros kept)
                x[j] = make_float2(__uint_as_float(u[j] << 16), __uint_as_float(u[j] & 0xFFFF0000u));
            if (IS_K) {
                // RN(K - mean)
#pragma unroll
                for (int k = 0; k < 4; ++k) {
                    const float4 m = __ldg(mp + k);
                    x[2 * k] = __fadd2_rn(x[2 * k], make_float2(-m.x, -m.y));
                    x[2 * k + 1] = __fadd2_rn(x[2 * k + 1], make_float2(-m.z, -m.w));
                }
            }
        }
        const float ab = fmaxf(max_abs8(x), max_abs8(x + 4));
        const BlockCodes16 bc = encode_block16(x, ab, tab, c, a.one);
        if (full || 4 * it < nt) *dst = bc.q;
        dst += 32;
        *sbw = (uint8_t)bc.sb;
        sbw += 32;
    }
    __syncwarp();
    if (lane < kEncTokens && t0 + lane < a.T) {
        uint8_t* scales = IS_K ? a.k_scales : a.v_scales;
        *reinterpret_cast<uint2*>(scales + ((size_t)h * a.T + t0 + lane) * 8) =
            *reinterpret_cast<const uint2*>(sbst + lane * 8);
    }
    __syncwarp();
}

// ---------------------------------------------------------------- finalize

// The mean and max |K - mean| of a 32-column block from every segment's
// statistics: the NSW statistics warps (named barrier 1) stage the segments in
// shared memory, warp 0 adds them in segment order.  Returns
// (in warp 0) the block's max |K - mean|.
template <int NSW>
__device__ float finalize_block(const QuantArgs& a, QuantShared& sh, int b) {
    constexpr int kSegsPerStatsWarp = kFinSegs / NSW;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int col = b * kFinCols + lane;
    const unsigned short* pmin = reinterpret_cast<const unsigned short*>(a.pmin);
    const unsigned short* pmax = reinterpret_cast<const unsigned short*>(a.pmax);
    float S = 0.0f, mn = INFINITY, mx = -INFINITY;
    for (int s0 = 0; s0 < a.nseg; s0 += kFinSegs) {
        const int ns = min(kFinSegs, a.nseg - s0);
        float ps[kSegsPerStatsWarp];
        unsigned short pn[kSegsPerStatsWarp], px[kSegsPerStatsWarp];
#pragma unroll
        for (int j = 0; j < kSegsPerStatsWarp; ++j) {
            const int k = warp + j * NSW;
            if (k < ns) {
                const size_t i = (size_t)(s0 + k) * a.HD + col;
                ps[j] = __ldcg(a.psum + i);
                pn[j] = __ldcg(pmin + i);
                px[j] = __ldcg(pmax + i);
            }
        }
#pragma unroll
        for (int j = 0; j < kSegsPerStatsWarp; ++j) {
            const int k = warp + j * NSW;
            if (k < ns) {
                sh.fsum[k][lane] = ps[j];
                sh.fmin[k][lane] = pn[j];
                sh.fmax[k][lane] = px[j];
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NSW * 32));
        if (warp == 0) {
            for (int k = 0; k < ns; ++k) {
                S = __fadd_rn(S, sh.fsum[k][lane]);
                mn = fminf(mn, __uint_as_float((uint32_t)sh.fmin[k][lane] << 16));
                mx = fmaxf(mx, __uint_as_float((uint32_t)sh.fmax[k][lane] << 16));
            }
        }
        asm volatile("bar.sync 1, %0;" ::"n"(NSW * 32));
    }
    float kp = 0.0f;
    if (warp == 0) {
        const float mu = __fdiv_rn(S, (float)a.T);
        a.k_mean[col] = mu;
        kp = fmaxf(fabsf(__fsub_rn(mx, mu)), fabsf(__fsub_rn(mn, mu)));
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) kp = fmaxf(kp, __shfl_xor_sync(0xFFFFFFFFu, kp, o));
    }
    return kp;
}

// The finalize of the sequence-parallel path: all warps of a CTA per 32-column
// block, the CTA's max |K - mean| into kpart[blockIdx.x].
__device__ void phase_finalize_all(const QuantArgs& a, QuantShared& sh) {
    float kp = 0.0f;
    const int nblocks = a.HD / kFinCols;
    const float Tf = (float)a.T;
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const unsigned short* pmin = reinterpret_cast<const unsigned short*>(a.pmin);
    const unsigned short* pmax = reinterpret_cast<const unsigned short*>(a.pmax);
    constexpr int kPer = kFinSegs / kQuantWarps;
    for (int b = blockIdx.x; b < nblocks; b += gridDim.x) {
        const int col = b * kFinCols + lane;
        float S = 0.0f, mn = INFINITY, mx = -INFINITY;
        for (int s0 = 0; s0 < a.nseg; s0 += kFinSegs) {
            const int ns = min(kFinSegs, a.nseg - s0);
            float ps[kPer];
            unsigned short pn[kPer], px[kPer];
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int k = warp + j * kQuantWarps;
                if (k < ns) {
                    const size_t i = (size_t)(s0 + k) * a.HD + col;
                    ps[j] = __ldcg(a.psum + i);
                    pn[j] = __ldcg(pmin + i);
                    px[j] = __ldcg(pmax + i);
                }
            }
#pragma unroll
            for (int j = 0; j < kPer; ++j) {
                const int k = warp + j * kQuantWarps;
                if (k < ns) {
                    sh.fsum[k][lane] = ps[j];
                    sh.fmin[k][lane] = pn[j];
                    sh.fmax[k][lane] = px[j];
                }
            }
            __syncthreads();
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

// ---------------------------------------------------------------- the kernel

// CTA 0 records when it starts and when it passes a few milestones (its first
// thread, or the warp that reaches them): a per-phase profile of the launch.
__device__ __forceinline__ void stamp(const QuantArgs& a, int i) {
    if (blockIdx.x == 0) a.ctl->stamp[i] = globaltimer_ns();
}

// A warp takes the next item of a CTA queue: index i < n, or -1.
__device__ __forceinline__ int take(unsigned* q, int n, volatile int* abort) {
    int i = 0;
    if ((threadIdx.x & 31) == 0) i = *abort ? n : (int)atomicAdd(q, 1u);
    i = __shfl_sync(0xFFFFFFFFu, i, 0);
    return i < n ? i : -1;
}

template <bool ROPE>
__global__ void __launch_bounds__(kQuantThreads, 1) quantize_kernel(QuantArgs a) {
    __shared__ QuantShared sh;
    extern __shared__ float2 rope_sm[];           // ROPE: the staged rotation table
    if (ROPE) rope_stage(a.rope, rope_sm);        // published by phase_vmax's barriers
    const uint64_t keep = policy_keep(), release = policy_release();
    const int lane = threadIdx.x & 31;
    const int warp = threadIdx.x >> 5;
    const int G = gridDim.x, b = blockIdx.x;
    if (threadIdx.x == 0) {
        sh.ready[0] = sh.ready[1] = 0;
        sh.claim[0] = sh.claim[1] = 0;
        sh.abort = 0;
        sh.q_stats = sh.q_v = sh.q_k = 0u;
        stamp(a, 0);
    }
    // 1. max |V| (its barriers also publish the initialization above)
    const float vmax = phase_vmax(a, sh, keep);
    if (threadIdx.x == 0) {
        atomicMax(&a.ctl->q_vmax, __float_as_uint(vmax));
        __threadfence();
        atomicAdd(&a.ctl->q_vdone, 1u);
        stamp(a, 1);
    }
    // even slices of every kind of unit per CTA
    const int n_stats = a.nseg * a.ngroups;
    const int s0 = (int)((long long)n_stats * b / G), s1 = (int)((long long)n_stats * (b + 1) / G);
    const int tiles = (a.T + kEncTokens - 1) / kEncTokens;
    const int n_units = a.H * tiles;
    const int u0 = (int)((long long)n_units * b / G), u1 = (int)((long long)n_units * (b + 1) / G);
    volatile int* abort = &sh.abort;
    uint8_t* sbst = sh.sb[warp];

    constexpr int NSW = ROPE ? kStatsWarpsRope : kStatsWarps;
    if (warp < NSW) {
        // 2a. K statistics from HBM
        int done = 0;
        for (int i; (i = take(&sh.q_stats, s1 - s0, abort)) >= 0; ++done)
            stats_unit<ROPE>(a, rope_sm, s0 + i, keep);
        __threadfence();
        if (lane == 0 && done > 0) atomicAdd(&a.ctl->q_sdone, (unsigned)done);
        // 2b. this CTA's column blocks, once every CTA's statistics are in
        const int nfin = a.HD / kFinCols;
        for (int fb = b; fb < nfin; fb += G) {
            // thread 0 decides for all statistics warps (a later abort by another
            // warp must not split them across the named barriers below)
            if (threadIdx.x == 0)
                sh.fin_go = wait_counter(&a.ctl->q_sdone, (unsigned)n_stats, a.ctl, abort, 106u);
            asm volatile("bar.sync 1, %0;" ::"n"(NSW * 32));
            if (!sh.fin_go) break;
            const float kp = finalize_block<NSW>(a, sh, fb);
            if (warp == 0 && lane == 0) {
                atomicMax(&a.ctl->q_kmax, __float_as_uint(kp));
                __threadfence();
                atomicAdd(&a.ctl->q_fdone, 1u);
            }
        }
        if (warp == 0 && lane == 0) stamp(a, 2);
    }
    // 2c. V from L2
    if (ensure_table(a, sh, 0)) {
        if (warp == NSW && lane == 0) stamp(a, 3);
        const EncodeConsts c = encode_consts(sh.s[0]);
        for (int i; (i = take(&sh.q_v, u1 - u0, abort)) >= 0;) {
            const int u = u0 + i;
            const int h = u / tiles;
            encode_unit<false, false>(a, sh.tab[0], c, sbst, h, (u - h * tiles) * kEncTokens,
                                      release);
        }
    }
    // 3. K from L2
    if (ensure_table(a, sh, 1)) {
        if (lane == 0) stamp(a, 4);
        const EncodeConsts c = encode_consts(sh.s[1]);
        for (int i; (i = take(&sh.q_k, u1 - u0, abort)) >= 0;) {
            const int u = u0 + i;
            const int h = u / tiles;
            encode_unit<true, ROPE>(a, sh.tab[1], c, sbst, h, (u - h * tiles) * kEncTokens,
                                    release, rope_sm);
        }
    }
    __syncthreads();
    if (threadIdx.x == 0) {
        stamp(a, 5);
        __threadfence();
        if (atomicAdd(&a.ctl->q_exit, 1u) == (unsigned)G - 1u) {
            // the last CTA: every other CTA is done with the counters
            a.ctl->q_vdone = 0u;
            a.ctl->q_vmax = 0u;
            a.ctl->q_sdone = 0u;
            a.ctl->q_fdone = 0u;
            a.ctl->q_kmax = 0u;
            __threadfence();
            a.ctl->q_exit = 0u;
        }
    }
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
    for (int u = wg; u < a.nseg * a.ngroups; u += nw) stats_unit<false>(a, nullptr, u, keep);
    const float b = phase_vmax(a, sh, keep);         // per-CTA max |V| ...
    if (threadIdx.x == 0) atomicMax(vmax_bits, __float_as_uint(b));
}

__global__ void __launch_bounds__(kQuantThreads, 1) sp_finalize_kernel(QuantArgs a) {
    __shared__ QuantShared sh;
    phase_finalize_all(a, sh);               // k_mean, per-CTA max |K - mean| in kpart
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
    fill_table(sh.tab[0], st, threadIdx.x, blockDim.x);
    __syncthreads();
    const EncodeConsts c = encode_consts(st);
    const uint64_t release = policy_release();
    const int warp = threadIdx.x >> 5;
    const int wg = blockIdx.x * kQuantWarps + warp;
    const int nw = gridDim.x * kQuantWarps;
    const int tiles = (a.T + kEncTokens - 1) / kEncTokens;
    for (int u = wg; u < a.H * tiles; u += nw) {
        const int h = u / tiles;
        const int t0 = (u - h * tiles) * kEncTokens;
        if (isK)
            encode_unit<true, false>(a, sh.tab[0], c, sh.sb[warp], h, t0, release);
        else
            encode_unit<false, false>(a, sh.tab[0], c, sh.sb[warp], h, t0, release);
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

int g_quant_grid[2][64];   // cooperative grid size per kernel and device ordinal (0: unknown)

}  // namespace

nvfp4kv_status launch_quantize(const void* K, const void* V, int T, int H,
                               const nvfp4kv_chunk_view& out, void* ws, cudaStream_t stream,
                               const RopeGeom* rope) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4KV_ERR_CUDA;
    const void* kernel = rope ? (const void*)quantize_kernel<true> : (const void*)quantize_kernel<false>;
    int& grid = g_quant_grid[rope ? 1 : 0][dev];
    if (grid == 0) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4KV_ERR_CUDA;
        const size_t dyn = rope ? kRopeMaxStagedBytes : 0;
        if (rope && cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)dyn) != cudaSuccess)
            return NVFP4KV_ERR_CUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kQuantThreads, dyn) !=
                cudaSuccess ||
            per_sm < 1)
            return NVFP4KV_ERR_CUDA;
        grid = min(sms * per_sm, kMaxGrid);
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
    a.rope = rope ? rope_dev(*rope) : RopeDev{};
    void* args[] = {&a};
    const size_t smem = rope ? rope_staged_bytes(rope->frames, rope->rows, rope->cols) : 0;
    cudaError_t e = cudaLaunchCooperativeKernel(kernel, dim3(grid), dim3(kQuantThreads), args,
                                                smem, stream);
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
