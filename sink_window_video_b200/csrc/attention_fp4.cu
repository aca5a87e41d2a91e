// attention_fp4.cu -- sink-window attention with an FP4-operand Q K^T: the
// queries quantized to NVFP4 and S = Q_hat K_hat^T taken by the block-scaled
// tcgen05 MMA (kind::mxf4nvf4) straight from the cache's E2M1 codes and E4M3
// block scales; P V as in attention_ws.cu (fp16 P in tensor memory, V
// de-quantized to exact fp16 in shared memory).
//
// Method ("2605-LongLive2" DeepRead page, Method > 推理基础设施: on Blackwell
// the generator runs W4A4, FP4 GEMMs in place of BF16 ones; Method >
// 训练基础设施: activations in 1D NVFP4 blocks with Four-Over-Six): Q [T_q, H,
// d] is quantized as the matrix [T_q * H, d] (16-element blocks along d, one
// FP32 tensor scale s_Q) by the weight / activation quantizer, then
//   S = s_Q s_K (sum over blocks of (q_Q sb_Q)(q_K sb_K)) + Q_hat . mean_c,
// the block products summed by the tensor core in fp32.  The output is
// attention with the queries replaced by their NVFP4 reconstruction.
//
// One CTA per SM: a head and 256 query rows (two 128-row tiles), keys in
// 96-key tiles (the scale-factor layout wants N in multiples of 32, and
// 2 x 96 S columns leave tensor memory for the scale factors):
//   warps 0-7   softmax (thread = row = tensor-memory lane), tile qi = warp / 4;
//               at the start they stage their tile's FP4 Q and Q scales
//   warp 8      the MMA issue (lane 0) and lane quarter 0 of the K scales
//   warps 9-11  producers: per key tile, thread j copies key row j's codes into
//               the FP4 operand layout and de-quantizes value row j to fp16;
//               each warp writes its lane quarter of the K scales
// Tensor memory (512 columns): S0 0..95 | Q scales 96..111 | S1 128..223 |
// K scales 224..247 (three ring stages) | O0 256..383 | O1 384..511.  A
// block-scaled operand's scale factors for 128 (or 96) rows and one K = 64
// step take 4 columns: row r in column r / 32 at lane r % 32 of every lane
// quarter, byte = 16-element block.
// Shared memory: Q tiles (FP4, 2 x 8 KB), a three-stage ring of K code tiles
// (FP4, 6 KB) and V tiles (fp16, 24 KB, 128-byte swizzle, MN-major), and one
// P tile per query tile (fp16, 24 KB).  The FP4 operands and P use the
// no-swizzle K-major layout: 16-byte chunk c of row r at (r / 8) SBO + c 128 +
// (r % 8) 16 (SBO 512 for 64-byte rows, 1536 for P's 192-byte rows).
// Because P lives in shared memory, S is free as soon as the softmax has read
// it: per key tile t the MMA warp issues QK_i(t+1) once tile i has read S_i(t)
// (s_free), then PV_i(t) once P_i(t) is written (p_full).  The next tile's
// logits are therefore ready while this tile's exponentials are computed; the
// softmax waits for PV_i(t-1) (pv_done) only before it rescales O_i or
// overwrites P_i.
// Waits, abort path and work split are attention_ws.cu's.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace nvfp4kv {
using namespace tc;
namespace {

constexpr int kKeysF = 96;                   // keys per tile
constexpr int kStagesF = 3;
constexpr int kThreadsF = 384;
constexpr int kMmaWarpF = 8;
constexpr int kProdWarp0 = 9;
__device__ __forceinline__ uint32_t col_s(int qi) { return 128u * (uint32_t)qi; }   // S of tile qi
constexpr uint32_t kColSFA = 96;             // + 8 qi + 4 s
constexpr uint32_t kColSFB = 224;            // + 8 stage + 4 s
constexpr uint32_t kColO = 256;              // + 128 qi
constexpr uint32_t kColsF = 512;
constexpr int kQTileB = 128 * 64;            // FP4 Q tile (128 rows x 64 B)
constexpr int kKTileB = kKeysF * 64;         // FP4 K tile (96 rows x 64 B)
constexpr int kVHalfB = kKeysF * 128;        // one 64-channel half of a V tile
constexpr int kVTileB = 2 * kVHalfB;         // fp16 V tile (96 rows x 256 B)
constexpr int kOffK = 2 * kQTileB;
constexpr int kOffV = 34 * 1024;             // 1024-byte aligned (128-byte swizzle atoms)
static_assert(kOffK + kStagesF * kKTileB <= kOffV, "K ring fits below the V ring");
constexpr int kPTileB = 128 * kKeysF * 2;    // fp16 P of one query tile (128 rows x 96 keys)
constexpr int kOffP = kOffV + kStagesF * kVTileB;          // 106 KB
static_assert(kOffP % 1024 == 0, "P tiles aligned");
constexpr size_t kSmemF = kOffP + 2 * (size_t)kPTileB + 1024;
constexpr float kLog2eF = 1.4426950408889634f;
constexpr float kRescaleLog2F = 8.0f;
constexpr float kFarLog2F = 48.0f;
constexpr float kRangeLog2F = 116.0f;

struct FChunk {
    const uint8_t* k_codes;
    const uint8_t* k_scales;
    const uint8_t* v_codes;
    const uint8_t* v_scales;
    const float* k_mean;
    const float* tensor_scales;
};

struct FArgs {
    FChunk chunk[NVFP4KV_MAX_KEY_CHUNKS];
    int n_chunks, T_c, H, T_q;
    const uint8_t* q_codes;      // [T_q * H][64]
    const uint8_t* q_scales;     // [T_q * H][8]
    const float* q_scale;        // s_Q
    void* O;
    int o_f32;
    float scale_log2;
    Control* ctl;
    int pairs_per_head, n_full, n_split;
    float* part;
};

struct FShared {
    uint64_t kv_full[kStagesF];
    uint64_t kv_empty[kStagesF];
    uint64_t s_full[2];
    uint64_t s_free[2];      // every row of tile qi has read its S
    uint64_t p_full[2];
    uint64_t pv_done[2];     // one phase per P V of tile qi
    uint64_t q_ready[2];
    uint64_t o_final;
    uint64_t drain;
    uint32_t tmem_base;
    int abort;
};

__device__ __forceinline__ uint32_t core_off(int r, int c) {
    return (uint32_t)((r >> 3) * 512 + c * 128 + (r & 7) * 16);
}

// Byte offset of 16-byte chunk c (0..15 along d) of key row r in a V tile:
// [2 halves of 64 channels][96 rows][128 B], 128-byte swizzle.
__device__ __forceinline__ uint32_t v_off(int r, int c) {
    return (uint32_t)((c >> 3) * kVHalfB + r * 128 + (((c & 7) ^ (r & 7)) << 4));
}

__device__ __forceinline__ bool wait_or_abort_f(uint32_t mbar, uint32_t parity, volatile int* abort,
                                                Control* ctl, unsigned site, unsigned step) {
    if (mbar_try_wait(mbar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    while (true) {
#pragma unroll 1
        for (int i = 0; i < 16; ++i)
            if (mbar_try_wait(mbar, parity)) return true;
        if (*abort) return false;
        if (globaltimer_ns() - t0 > kWaitLimitNs) {
            *abort = 1;
            record_timeout(ctl, site, step, parity);
            return false;
        }
    }
}

// One value row (64 code bytes, 8 E4M3 scale bytes) to fp16 q*sb, into row r
// of a V tile.
__device__ __forceinline__ void dequant_v_row(const uint4* cw4, uint2 sc, uint8_t* tile, int r) {
    const uint32_t sp[4] = {cvt_e4m3x2_to_f16x2(sc.x & 0xFFFFu), cvt_e4m3x2_to_f16x2(sc.x >> 16),
                            cvt_e4m3x2_to_f16x2(sc.y & 0xFFFFu), cvt_e4m3x2_to_f16x2(sc.y >> 16)};
#pragma unroll
    for (int b = 0; b < 8; ++b) {
        const uint32_t pair = sp[b >> 1];
        const uint32_t shv = (b & 1) ? (pair >> 16) : (pair & 0xFFFFu);
        const uint32_t s2 = shv | (shv << 16);
#pragma unroll
        for (int w = 0; w < 2; ++w) {
            const uint32_t word = (&cw4[b >> 1].x)[(b & 1) * 2 + w];
            uint32_t hh[4];
            cvt_e2m1x8_to_f16x2(word, hh);
            uint4 o;
            o.x = hmul2_u32(hh[0], s2);
            o.y = hmul2_u32(hh[1], s2);
            o.z = hmul2_u32(hh[2], s2);
            o.w = hmul2_u32(hh[3], s2);
            *reinterpret_cast<uint4*>(tile + v_off(r, 2 * b + w)) = o;
        }
    }
}

__device__ __forceinline__ float fmax3f(float a, float b, float c) {
    float d;
    asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
    return d;
}

// The K scale words of one key tile for this lane's rows (lane, 32 + lane,
// 64 + lane) and both K = 64 steps; zeros past the chunk's end.
struct SfbRows {
    uint2 w[3];
};
__device__ __forceinline__ SfbRows load_sfb(const FArgs& a, int h, int gt, int tiles_per_chunk,
                                            int lane, bool valid_tile) {
    SfbRows r;
    const int ci = gt / tiles_per_chunk;
    const int k0 = (gt - ci * tiles_per_chunk) * kKeysF;
#pragma unroll
    for (int j = 0; j < 3; ++j) {
        const int key = k0 + 32 * j + lane;
        r.w[j] = (valid_tile && key < a.T_c)
                     ? *reinterpret_cast<const uint2*>(a.chunk[ci].k_scales +
                                                       ((size_t)h * a.T_c + key) * 8)
                     : make_uint2(0u, 0u);
    }
    return r;
}
__device__ __forceinline__ void store_sfb(uint32_t tmem, uint32_t lane_base, int st, const SfbRows& r) {
    const uint32_t w0[4] = {r.w[0].x, r.w[1].x, r.w[2].x, 0u};
    const uint32_t w1[4] = {r.w[0].y, r.w[1].y, r.w[2].y, 0u};
    tmem_st4(tmem + lane_base + kColSFB + 8u * st, w0);
    tmem_st4(tmem + lane_base + kColSFB + 8u * st + 4u, w1);
}

__global__ void __launch_bounds__(kThreadsF, 1) attention_fp4_kernel(const FArgs a) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ FShared sh;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int lane = tid & 31;
    const int item = blockIdx.x;
    const bool split = item >= a.n_full;
    const int piece = split ? item - a.n_full : 0;
    const int pair = split ? a.n_full + piece / a.n_split : item;
    const int q_split = split ? piece % a.n_split : 0;
    const int n_ranges = split ? a.n_split : 1;
    const int h = pair / a.pairs_per_head;
    const int m0 = (pair - h * a.pairs_per_head) * 256;
    const int H = a.H, T_c = a.T_c;
    const int tiles_per_chunk = (T_c + kKeysF - 1) / kKeysF;
    const int ntiles_all = a.n_chunks * tiles_per_chunk;
    const int t_begin = (int)((long long)ntiles_all * q_split / n_ranges);
    const int ntiles = (int)((long long)ntiles_all * (q_split + 1) / n_ranges) - t_begin;
    volatile int* abort = &sh.abort;

    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* Qt = base;
    uint8_t* Kt = base + kOffK;
    uint8_t* Vt = base + kOffV;
    uint8_t* Pt = base + kOffP;                  // [2][P tile], no-swizzle K-major core matrices

    if (warp == kMmaWarpF) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&sh.tmem_base)),
                     "r"(kColsF));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        sh.abort = 0;
        for (int s = 0; s < kStagesF; ++s) {
            mbar_init(smem_u32(&sh.kv_full[s]), 32 * 3);
            mbar_init(smem_u32(&sh.kv_empty[s]), 1);
        }
        for (int i = 0; i < 2; ++i) {
            mbar_init(smem_u32(&sh.s_full[i]), 1);
            mbar_init(smem_u32(&sh.s_free[i]), 128);
            mbar_init(smem_u32(&sh.p_full[i]), 128);
            mbar_init(smem_u32(&sh.pv_done[i]), 1);
            mbar_init(smem_u32(&sh.q_ready[i]), 128);
        }
        mbar_init(smem_u32(&sh.o_final), 1);
        mbar_init(smem_u32(&sh.drain), 1);
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = sh.tmem_base;

    if (warp < 8) {
        // ------------------------------------------------------------ softmax
        const int qi = warp >> 2;
        const int r = tid & 127;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        const uint32_t tS = tmem + lane_base + col_s(qi);
        const uint32_t tO = tmem + lane_base + kColO + 128u * qi;
        const int row = m0 + qi * 128 + r;
        const bool rvalid = row < a.T_q;
        const size_t qrow = (size_t)row * H + h;
        const float sQ = *a.q_scale;

        // this row's FP4 codes into the Q tile; the Q scales of this lane's
        // rows (lane, 32 + lane, 64 + lane, 96 + lane) into tensor memory
        {
            const uint4* qc = reinterpret_cast<const uint4*>(a.q_codes + qrow * 64);
            uint8_t* qt = Qt + qi * kQTileB;
#pragma unroll
            for (int c = 0; c < 4; ++c)
                *reinterpret_cast<uint4*>(qt + core_off(r, c)) =
                    rvalid ? qc[c] : make_uint4(0u, 0u, 0u, 0u);
            uint32_t s0[4], s1[4];
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                const int rr = m0 + qi * 128 + 32 * j + lane;
                const uint2 w = rr < a.T_q ? *reinterpret_cast<const uint2*>(
                                                 a.q_scales + ((size_t)rr * H + h) * 8)
                                           : make_uint2(0u, 0u);
                s0[j] = w.x;
                s1[j] = w.y;
            }
            tmem_st4(tmem + lane_base + kColSFA + 8u * qi, s0);
            tmem_st4(tmem + lane_base + kColSFA + 8u * qi + 4u, s1);
            tmem_wait_st();
        }
        fence_async_smem();
        tc_fence_before();
        mbar_arrive(smem_u32(&sh.q_ready[qi]));

        auto log2_svmax = [&]() {
            float v = 0.0f;
            for (int ci = 0; ci < a.n_chunks; ++ci) v = fmaxf(v, a.chunk[ci].tensor_scales[1]);
            return log2f(v);
        };

        float m_run = -INFINITY, l_run = 0.0f;
        bool o_written = false, ok = true;
        int t = 0;
        const uint32_t s_full = smem_u32(&sh.s_full[qi]);
        const uint32_t p_full = smem_u32(&sh.p_full[qi]);
        int ci_cur = -1;
        float alpha = 0.0f, beta = 0.0f, lrV = 0.0f, inv_rV = 0.0f;
        float2 alpha2 = make_float2(0.0f, 0.0f);
        for (; t < ntiles && ok; ++t) {
            const int gt = t_begin + t;
            const int ci = gt / tiles_per_chunk;
            const int j0 = (gt - ci * tiles_per_chunk) * kKeysF;
            if (ci != ci_cur) {
                ci_cur = ci;
                const FChunk cp = a.chunk[ci];
                const float sK = cp.tensor_scales[0], sV = cp.tensor_scales[1];
                // Q_hat . mean of this chunk: Q_hat = decode(q) decode(sb) s_Q
                float qmu = 0.0f;
                if (rvalid) {
                    const uint4* qc = reinterpret_cast<const uint4*>(a.q_codes + qrow * 64);
                    const uint2 qs = *reinterpret_cast<const uint2*>(a.q_scales + qrow * 8);
                    const float4* mp = reinterpret_cast<const float4*>(cp.k_mean + h * kHeadDim);
#pragma unroll 1
                    for (int b = 0; b < 8; ++b) {
                        const uint4 cw = qc[b >> 1];
                        const uint32_t w0 = (b & 1) ? cw.z : cw.x, w1 = (b & 1) ? cw.w : cw.y;
                        uint32_t hh[8];
                        cvt_e2m1x8_to_f16x2(w0, hh);
                        cvt_e2m1x8_to_f16x2(w1, hh + 4);
                        float blk = 0.0f;
#pragma unroll
                        for (int k = 0; k < 4; ++k) {
                            const float4 u = mp[4 * b + k];
                            blk = fmaf(f16lo(hh[2 * k]), u.x, blk);
                            blk = fmaf(f16hi(hh[2 * k]), u.y, blk);
                            blk = fmaf(f16lo(hh[2 * k + 1]), u.z, blk);
                            blk = fmaf(f16hi(hh[2 * k + 1]), u.w, blk);
                        }
                        const uint32_t sbyte = ((b < 4 ? qs.x : qs.y) >> (8 * (b & 3))) & 0xFFu;
                        qmu = fmaf(e4m3_to_f32(sbyte), blk, qmu);
                    }
                    qmu *= sQ;
                }
                alpha = sQ * sK * a.scale_log2;
                lrV = fmaxf(log2f(sV) - log2_svmax(), -126.0f);
                beta = fmaf(qmu, a.scale_log2, lrV);
                inv_rV = ex2f(-lrV);
                alpha2 = make_float2(alpha, alpha);
                if (lrV < -kRangeLog2F && r == 0 && (warp & 3) == 0)
                    atomicOr(&a.ctl->status, kStatusRange);
            }
            {
                bool got = wait_or_abort_f(s_full, (uint32_t)(t & 1), abort, a.ctl, 10u + qi, t);
                if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                tc_fence_after();
                const int valid = min(kKeysF, T_c - j0);
                // the whole S row, then S is free for the next tile's Q K^T
                uint32_t s[kKeysF];
                tmem_ld32(tS, s);
                tmem_ld32(tS + 32, s + 32);
                tmem_ld32(tS + 64, s + 64);
                tmem_wait_ld();
                tc_fence_before();
                mbar_arrive(smem_u32(&sh.s_free[qi]));
                if (valid < kKeysF) {
#pragma unroll
                    for (int k = 0; k < kKeysF; ++k)
                        if (k >= valid) s[k] = __float_as_uint(-INFINITY);
                }
                float m8[8];
#pragma unroll
                for (int c = 0; c < 8; ++c)
                    m8[c] = fmax3f(__uint_as_float(s[c]), __uint_as_float(s[c + 8]),
                                   __uint_as_float(s[c + 16]));
#pragma unroll
                for (int k = 24; k < kKeysF; k += 24)
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        m8[c] = fmax3f(m8[c], __uint_as_float(s[k + c]),
                                       fmax3f(__uint_as_float(s[k + 8 + c]), __uint_as_float(s[k + 16 + c]),
                                              m8[c]));
                float mx = fmax3f(fmax3f(m8[0], m8[1], m8[2]), fmax3f(m8[3], m8[4], m8[5]),
                                  fmaxf(m8[6], m8[7]));
                mx = fmaf(mx, alpha, beta);
                const bool grow = mx > m_run + kRescaleLog2F || (m_run == -INFINITY && mx > -INFINITY);
                float corr = 1.0f;
                if (grow) {
                    const float m_new = fmaxf(mx, m_run);
                    corr = ex2f(m_run - m_new);
                    l_run *= corr;
                    m_run = m_new;
                }
                if (lrV < -kFarLog2F) {
                    // (rare, chunk-uniform) the denominator from the keys' own
                    // exponentials
                    const float bl = beta - lrV - m_run;
                    float al = 0.0f;
#pragma unroll
                    for (int k = 0; k < kKeysF; ++k)
                        if (k < valid) al += ex2f(fmaf(__uint_as_float(s[k]), alpha, bl));
                    l_run += al;
                }
                const float b2 = beta - m_run;
                const float2 b22 = make_float2(b2, b2);
                float2 acc[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                                 make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f)};
                uint32_t p[kKeysF / 2];
#pragma unroll
                for (int k = 0; k < kKeysF / 2; ++k) {
                    float2 z = __ffma2_rn(make_float2(__uint_as_float(s[2 * k]), __uint_as_float(s[2 * k + 1])),
                                          alpha2, b22);
                    if ((k & 7) >= 6) {
                        z = ex2_poly2(z);
                    } else {
                        z.x = ex2f(z.x);
                        z.y = ex2f(z.y);
                    }
                    acc[k & 3] = __fadd2_rn(acc[k & 3], z);
                    p[k] = pack_f16x2(z.x, z.y);
                }
                if (!(lrV < -kFarLog2F)) {
                    const float2 a01 = __fadd2_rn(acc[0], acc[1]), a23 = __fadd2_rn(acc[2], acc[3]);
                    const float2 a03 = __fadd2_rn(a01, a23);
                    l_run += (a03.x + a03.y) * inv_rV;
                }
                // the previous P V is complete before O is rescaled and P is
                // overwritten
                if (t > 0) {
                    got = wait_or_abort_f(smem_u32(&sh.pv_done[qi]), (uint32_t)((t - 1) & 1), abort,
                                          a.ctl, 13u + qi, t);
                    if (!__all_sync(0xFFFFFFFFu, got)) { ok = false; break; }
                    tc_fence_after();
                }
                if (__any_sync(0xFFFFFFFFu, grow) && o_written) {
#pragma unroll 1
                    for (int q = 0; q < 4; ++q) {
                        uint32_t ov[32];
                        tmem_ld32(tO + 32 * q, ov);
                        tmem_wait_ld();
#pragma unroll
                        for (int i = 0; i < 32; ++i)
                            ov[i] = __float_as_uint(__uint_as_float(ov[i]) * corr);
                        tmem_st32(tO + 32 * q, ov);
                    }
                    tmem_wait_st();
                }
                // P' to this tile's P buffer: 16-byte chunk c (keys 8c .. 8c + 7)
                // of row r at (r / 8) 1536 + c 128 + (r % 8) 16
                uint8_t* prow = Pt + qi * kPTileB + (r >> 3) * 1536 + (r & 7) * 16;
#pragma unroll
                for (int c = 0; c < kKeysF / 8; ++c)
                    *reinterpret_cast<uint4*>(prow + c * 128) =
                        make_uint4(p[4 * c], p[4 * c + 1], p[4 * c + 2], p[4 * c + 3]);
                fence_async_smem();
                tc_fence_before();
                mbar_arrive(p_full);
                o_written = true;
            }
        }
        if (ok) {
            bool got = wait_or_abort_f(smem_u32(&sh.o_final), 0u, abort, a.ctl, 20u + qi, ntiles);
            ok = __all_sync(0xFFFFFFFFu, got);
        }
        if (ok) {
            tc_fence_after();
            float sVmax = 0.0f;
            for (int ci = 0; ci < a.n_chunks; ++ci) sVmax = fmaxf(sVmax, a.chunk[ci].tensor_scales[1]);
            const float inv = sVmax / l_run;
            float* prow = split ? a.part + ((size_t)piece * 256 + qi * 128 + r) * kPartialFloats
                                : nullptr;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
                uint32_t ov[32];
                __syncwarp();
                tmem_ld32(tO + 32 * q, ov);
                tmem_wait_ld();
                if (rvalid && split) {
                    float4* dst = reinterpret_cast<float4*>(prow + 32 * q);
#pragma unroll
                    for (int c = 0; c < 8; ++c)
                        dst[c] = make_float4(__uint_as_float(ov[4 * c]), __uint_as_float(ov[4 * c + 1]),
                                             __uint_as_float(ov[4 * c + 2]), __uint_as_float(ov[4 * c + 3]));
                } else if (rvalid) {
                    const size_t o = ((size_t)row * H + h) * kHeadDim + 32 * q;
                    if (a.o_f32) {
                        float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.O) + o);
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            dst[c] = make_float4(__uint_as_float(ov[4 * c]) * inv, __uint_as_float(ov[4 * c + 1]) * inv,
                                                 __uint_as_float(ov[4 * c + 2]) * inv, __uint_as_float(ov[4 * c + 3]) * inv);
                    } else {
                        uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.O) + o);
#pragma unroll
                        for (int c = 0; c < 4; ++c) {
                            uint32_t w4[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                __nv_bfloat162 b2v = __floats2bfloat162_rn(__uint_as_float(ov[8 * c + 2 * j]) * inv,
                                                                           __uint_as_float(ov[8 * c + 2 * j + 1]) * inv);
                                w4[j] = *reinterpret_cast<uint32_t*>(&b2v);
                            }
                            dst[c] = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                        }
                    }
                }
            }
            if (rvalid && split) {
                prow[128] = m_run;
                prow[129] = l_run / sVmax;
            }
        }
    } else if (warp >= kProdWarp0) {
        // ------------------------------------------------------------ producers
        // thread j (0..95) handles key row j of every tile: its K codes into
        // the FP4 operand layout and its value row to fp16; each warp also
        // writes its lane quarter of the tile's K scales.  The next tile's
        // row is loaded right after the current one is stored.
        const int j = tid - kProdWarp0 * 32;
        const uint32_t lane_base = (uint32_t)((warp & 3) * 32) << 16;
        // Test hook (bit 0 of the control block's test word, cleared by
        // workspace initialization): producer thread 0 of CTA 0 withholds its
        // first kv_full arrival, so that the waits behind it run out of time
        // and take the abort path.
        const bool withhold = blockIdx.x == 0 && j == 0 && (a.ctl->test_flags & 1u) != 0u;
        struct Row {
            uint4 kc[4];
            uint4 vc[4];
            uint2 vs;
        };
        auto load_row = [&](int tt, Row& rw, SfbRows& sf) {
            const int gt = t_begin + tt;
            const bool vt = tt < ntiles;
            const int ci = vt ? gt / tiles_per_chunk : 0;
            const int key = vt ? (gt - ci * tiles_per_chunk) * kKeysF + j : T_c;
            if (vt && key < T_c) {
                const FChunk& cp = a.chunk[ci];
                const size_t rowi = (size_t)h * T_c + key;
                const uint4* kp = reinterpret_cast<const uint4*>(cp.k_codes + rowi * 64);
                const uint4* vp = reinterpret_cast<const uint4*>(cp.v_codes + rowi * 64);
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    rw.kc[i] = kp[i];
                    rw.vc[i] = vp[i];
                }
                rw.vs = *reinterpret_cast<const uint2*>(cp.v_scales + rowi * 8);
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    rw.kc[i] = make_uint4(0, 0, 0, 0);
                    rw.vc[i] = make_uint4(0, 0, 0, 0);
                }
                rw.vs = make_uint2(0, 0);
            }
            sf = load_sfb(a, h, vt ? gt : 0, tiles_per_chunk, lane, vt);
        };
        Row rw;
        SfbRows sf;
        load_row(0, rw, sf);
        for (int t = 0; t < ntiles; ++t) {
            const int st = t % kStagesF;
            if (t >= kStagesF) {
                bool got = wait_or_abort_f(smem_u32(&sh.kv_empty[st]),
                                           (uint32_t)(((t / kStagesF) - 1) & 1), abort, a.ctl, 30u, t);
                if (!__all_sync(0xFFFFFFFFu, got)) break;
                tc_fence_after();
            }
            uint8_t* kt = Kt + st * kKTileB;
#pragma unroll
            for (int c = 0; c < 4; ++c) *reinterpret_cast<uint4*>(kt + core_off(j, c)) = rw.kc[c];
            dequant_v_row(rw.vc, rw.vs, Vt + st * kVTileB, j);
            store_sfb(tmem, lane_base, st, sf);
            load_row(t + 1, rw, sf);
            tmem_wait_st();
            fence_async_smem();
            tc_fence_before();
            if (!(withhold && t == 0)) mbar_arrive(smem_u32(&sh.kv_full[st]));
        }
    } else {
        // ------------------------------------------------------------ MMA issue (warp 8)
        // All lanes wait and write lane quarter 0 of each tile's K scales;
        // lane 0 issues.
        constexpr uint32_t idesc_qk = umma_idesc_fp4(kKeysF);
        constexpr uint32_t idesc_pv = umma_idesc_f16(true, 128);
        const uint64_t qdesc0 = umma_desc_noswizzle(smem_u32(Qt), 128, 512);
        const uint64_t kdesc0 = umma_desc_noswizzle(smem_u32(Kt), 128, 512);
        const uint64_t vdesc0 = umma_desc(smem_u32(Vt), kVHalfB, 1024);
        auto put_sfb = [&](int tt, const SfbRows& sf) {
            store_sfb(tmem, 0u, tt % kStagesF, sf);
            tmem_wait_st();
            tc_fence_before();
            __syncwarp();
            tc_fence_after();
        };
        auto issue_qk = [&](int qi, int st) {
            if (lane == 0) {
                const uint32_t dt = tmem + col_s(qi);
#pragma unroll
                for (int s = 0; s < 2; ++s) {
                    const uint64_t qd = qdesc0 + (uint64_t)((qi * kQTileB + 256 * s) >> 4);
                    const uint64_t kd = kdesc0 + (uint64_t)((st * kKTileB + 256 * s) >> 4);
                    mma_fp4(dt, qd, kd, idesc_qk, s > 0 ? 1u : 0u, tmem + kColSFA + 8u * qi + 4u * s,
                            tmem + kColSFB + 8u * st + 4u * s);
                }
                mma_commit(smem_u32(&sh.s_full[qi]));
            }
            __syncwarp();
        };
        // P V of tile qi: A = P (fp16, shared memory, no swizzle: LBO 128 along
        // the keys, SBO 1536 per 8 rows), B = V
        const uint64_t pdesc0 = umma_desc_noswizzle(smem_u32(Pt), 128, 1536);
        auto issue_pv = [&](int qi, int st, bool first) {
            if (lane == 0) {
                const uint64_t vd = vdesc0 + (uint64_t)((st * kVTileB) >> 4);
                const uint64_t pd = pdesc0 + (uint64_t)((qi * kPTileB) >> 4);
                const uint32_t dt = tmem + kColO + 128u * qi;
#pragma unroll
                for (int ks = 0; ks < kKeysF / 16; ++ks)
                    mma_ss(dt, pd + (uint64_t)((ks * 256) >> 4), vd + (uint64_t)((ks * 2048) >> 4),
                           idesc_pv, (ks > 0 || !first) ? 1u : 0u);
                mma_commit(smem_u32(&sh.pv_done[qi]));
            }
            __syncwarp();
        };
        auto wait_all = [&](uint64_t* bar, uint32_t parity, unsigned site, int step) {
            return __all_sync(0xFFFFFFFFu, wait_or_abort_f(smem_u32(bar), parity, abort, a.ctl,
                                                           site, (unsigned)step));
        };
        bool ok = wait_or_abort_f(smem_u32(&sh.q_ready[0]), 0u, abort, a.ctl, 40u, 0) &&
                  wait_or_abort_f(smem_u32(&sh.q_ready[1]), 0u, abort, a.ctl, 41u, 0);
        ok = __all_sync(0xFFFFFFFFu, ok);
        // lane quarter 0 of the K scales, loaded a tile ahead
        SfbRows sf_next = load_sfb(a, h, t_begin, tiles_per_chunk, lane, ntiles > 0);
        if (ok && ntiles > 0) {
            tc_fence_after();
            ok = wait_all(&sh.kv_full[0], 0u, 42u, 0);
            if (ok) {
                tc_fence_after();
                put_sfb(0, sf_next);
                issue_qk(0, 0);
                issue_qk(1, 0);
            }
        }
        // Per tile t: the next tile's Q K^T as soon as each query tile has read
        // its S, then this tile's P V as each P is written.
        for (int t = 0; t < ntiles && ok; ++t) {
            const int st = t % kStagesF;
            const bool more = t + 1 < ntiles;
            const int st2 = (t + 1) % kStagesF;
            sf_next = load_sfb(a, h, t_begin + t + 1, tiles_per_chunk, lane, more);
            if (more) {
                ok = wait_all(&sh.kv_full[st2], (uint32_t)(((t + 1) / kStagesF) & 1), 44u, t + 1);
                if (!ok) break;
                tc_fence_after();
                put_sfb(t + 1, sf_next);
            }
            for (int qi = 0; qi < 2 && ok; ++qi) {
                ok = wait_all(&sh.s_free[qi], (uint32_t)(t & 1), 46u + qi, t);
                if (!ok) break;
                tc_fence_after();
                if (more) issue_qk(qi, st2);
            }
            for (int qi = 0; qi < 2 && ok; ++qi) {
                ok = wait_all(&sh.p_full[qi], (uint32_t)(t & 1), 43u + 2 * qi, t);
                if (!ok) break;
                tc_fence_after();
                issue_pv(qi, st, t == 0);
            }
            if (!ok) break;
            if (lane == 0) mma_commit(smem_u32(&sh.kv_empty[st]));
            __syncwarp();
        }
        if (lane == 0) {
            if (ok) mma_commit(smem_u32(&sh.o_final));
            mma_commit(smem_u32(&sh.drain));
            const unsigned long long t0 = globaltimer_ns();
            while (!mbar_try_wait(smem_u32(&sh.drain), 0u) && globaltimer_ns() - t0 < kWaitLimitNs)
                __nanosleep(64);
        }
        __syncwarp();
    }

    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarpF) {
        __syncwarp();
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kColsF));
    }
}

}  // namespace

AttnPlan attention_fp4_plan(int n_chunks, int T_c, int H, int T_q, size_t tail_capacity_rows) {
    return attention_plan_tiles(n_chunks * ((T_c + kKeysF - 1) / kKeysF), H, T_q, 256,
                                tail_capacity_rows);
}

nvfp4kv_status launch_attention_fp4(const nvfp4kv_chunk_view* chunks, int n_chunks, int T_c,
                                    int H, const void* Q, int T_q, void* O, int o_dtype,
                                    float softmax_scale, void* q_fp4, void* ws,
                                    cudaStream_t stream) {
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(attention_fp4_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemF) != cudaSuccess)
            return NVFP4KV_ERR_CUDA;
        configured = true;
    }
    const WsLayout L = ws_layout(T_c, H);
    const Fp4qLayout F = fp4q_layout(T_q, H);
    char* qb = static_cast<char*>(q_fp4);
    // the queries as NVFP4 rows [T_q * H][d] (1D blocks along d, Four-Over-Six)
    uint8_t* q_codes = reinterpret_cast<uint8_t*>(qb + F.codes);
    uint8_t* q_scales = reinterpret_cast<uint8_t*>(qb + F.scales);
    float* q_scale = reinterpret_cast<float*>(qb + F.scale);
    nvfp4kv_status st = launch_quantize_matrix(Q, T_q * H, kHeadDim, NVFP4KV_BLOCKS_1D, q_codes,
                                               q_scales, q_scale, ws, stream);
    if (st != NVFP4KV_OK) return st;
    const AttnPlan plan = attention_fp4_plan(n_chunks, T_c, H, T_q, L.apart_rows);
    FArgs a;
    for (int i = 0; i < n_chunks; ++i) {
        a.chunk[i].k_codes = chunks[i].k_codes;
        a.chunk[i].k_scales = chunks[i].k_scales;
        a.chunk[i].v_codes = chunks[i].v_codes;
        a.chunk[i].v_scales = chunks[i].v_scales;
        a.chunk[i].k_mean = chunks[i].k_mean;
        a.chunk[i].tensor_scales = chunks[i].tensor_scales;
    }
    a.n_chunks = n_chunks;
    a.T_c = T_c;
    a.H = H;
    a.T_q = T_q;
    a.q_codes = q_codes;
    a.q_scales = q_scales;
    a.q_scale = q_scale;
    a.O = O;
    a.o_f32 = o_dtype == NVFP4KV_F32 ? 1 : 0;
    a.scale_log2 = softmax_scale * kLog2eF;
    a.ctl = static_cast<Control*>(ws);
    a.pairs_per_head = plan.blocks_per_head;
    a.n_full = plan.n_full;
    a.n_split = plan.n_split;
    a.part = reinterpret_cast<float*>(static_cast<char*>(ws) + L.apart);
    const int grid = plan.n_full + plan.n_tail * plan.n_split;
    attention_fp4_kernel<<<grid, kThreadsF, kSmemF, stream>>>(a);
    if (cudaGetLastError() != cudaSuccess) return NVFP4KV_ERR_CUDA;
    if (plan.n_tail > 0)
        return launch_attention_merge(a.part, plan, T_q, H, O, a.o_f32, stream);
    return NVFP4KV_OK;
}

}  // namespace nvfp4kv
