// attention_tc.cu -- sink-window attention over the NVFP4 cache on the sm_100a
// tensor cores (tcgen05 MMA, accumulators in tensor memory), with the
// de-quantization fused in shared memory.
//
// Method ("2605-LongLive2" DeepRead page, Method > 算法层设计: attention over
// K_eff = A_g u A_s u KV[t-W, t); Method > 推理基础设施: the NVFP4 cache is
// de-quantized inside the attention kernel):
//   O = softmax(scale Q K_hat^T) V_hat,  K_hat = q*sb*s_K + mean,  V_hat = q*sb*s_V.
//
// Exact operands: an E2M1 value times an E4M3 value has at most 6 significant
// bits and lies in [2^-10, 2688], so Kq = q*sb and Vq = q*sb are exact in
// fp16 (one cvt e2m1x2->f16x2 and one f16x2 multiply per two elements).  The
// per-chunk factors stay in fp32 outside the products:
//   Q K_hat^T = s_K (Q Kq^T) + (Q . mean_c)     a per-row, per-chunk bias
//   P V_hat   = s_Vmax (P (s_V/s_Vmax)) Vq       P scaled per chunk into [0, 256]
// Q is bf16; each row is scaled by a power of two 2^-e into fp16's range
// (exact for the row's significant values) and 2^e is folded into the logit
// scale.  Softmax statistics are fp32 with a base-2 exponent.
//
// Per CTA: one head, 128 query rows (thread i owns row i = TMEM lane i), the
// key chunks in 128-key tiles.  Per tile:
//   1. all threads de-quantize the K and V tiles into shared memory, laid out
//      as the 128-byte-swizzled operands the MMA reads (K: K-major B of
//      S = Q K^T; V: MN-major B of O += P V; the same physical layout);
//   2. thread 0 issues S = Q Kq^T (8 MMAs of K=16) into TMEM, commits to an
//      mbarrier;
//   3. each thread loads its S row from TMEM, updates the running max/sum,
//      writes P (fp16) back over the first 64 columns of S;
//   4. thread 0 issues O += P Vq with P read from TMEM (8 MMAs), commits.
// Two CTAs share an SM (256 TMEM columns and ~97 KB of shared memory each),
// so one CTA's softmax runs beside the other's MMAs.  The running max is
// raised lazily: O (in TMEM) is rescaled only when a row's max grows by more
// than 2^8.  Every mbarrier wait is bounded; on timeout the CTA records
// kStatusTimeout in the workspace, waits (bounded) for its MMAs, frees its
// tensor memory and returns.
#include "common.cuh"
#include "kernels.h"
#include "tc_ptx.cuh"

namespace nvfp4kv {
namespace {

constexpr int kRows = 128;
constexpr int kKeys = 128;
constexpr int kThreadsTc = 128;
constexpr uint32_t kTmemCols = 256;        // S / P: [0, 128), O: [128, 256)
constexpr uint32_t kOCol = 128;
constexpr int kTileBytes = kRows * kHeadDim * 2;   // 32 KB of fp16
constexpr size_t kSmemTc = 3 * kTileBytes + 1024 + 64;
constexpr float kLog2eTc = 1.4426950408889634f;
constexpr float kRescaleThreshold = 8.0f;  // log2 units

struct TcChunk {
    const uint8_t* k_codes;
    const uint8_t* k_scales;
    const uint8_t* v_codes;
    const uint8_t* v_scales;
    const float* k_mean;
    const float* tensor_scales;
};

struct TcArgs {
    TcChunk chunk[NVFP4KV_MAX_KEY_CHUNKS];
    int n_chunks, T_c, H, T_q;
    const uint16_t* Q;
    void* O;
    int o_f32;
    float scale_log2;
    Control* ctl;
};

}  // namespace
using namespace tc;
namespace {

// De-quantize one 128-channel row (64 code bytes, 8 scale bytes) to fp16 in
// the swizzled tile at `tile` (row r).
__device__ __forceinline__ void dequant_row(const uint8_t* codes, const uint8_t* scales,
                                            uint8_t* tile, int r) {
    const uint4* cp = reinterpret_cast<const uint4*>(codes);
    const uint2 sc = *reinterpret_cast<const uint2*>(scales);
    uint4 cw[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) cw[i] = cp[i];
    const uint32_t s01 = cvt_e4m3x2_to_f16x2(sc.x & 0xFFFFu);
    const uint32_t s23 = cvt_e4m3x2_to_f16x2(sc.x >> 16);
    const uint32_t s45 = cvt_e4m3x2_to_f16x2(sc.y & 0xFFFFu);
    const uint32_t s67 = cvt_e4m3x2_to_f16x2(sc.y >> 16);
    const uint32_t sp[4] = {s01, s23, s45, s67};
#pragma unroll
    for (int b = 0; b < 8; ++b) {      // block b: code words 2b, 2b+1 -> chunks 2b, 2b+1
        const uint32_t pair = sp[b >> 1];
        const uint32_t sh = (b & 1) ? (pair >> 16) : (pair & 0xFFFFu);
        const uint32_t s2 = sh | (sh << 16);
        const uint32_t w0 = (&cw[b >> 1].x)[(b & 1) * 2];
        const uint32_t w1 = (&cw[b >> 1].x)[(b & 1) * 2 + 1];
        uint32_t h0[4], h1[4];
        cvt_e2m1x8_to_f16x2(w0, h0);
        cvt_e2m1x8_to_f16x2(w1, h1);
        uint4 o0, o1;
        o0.x = hmul2_u32(h0[0], s2); o0.y = hmul2_u32(h0[1], s2);
        o0.z = hmul2_u32(h0[2], s2); o0.w = hmul2_u32(h0[3], s2);
        o1.x = hmul2_u32(h1[0], s2); o1.y = hmul2_u32(h1[1], s2);
        o1.z = hmul2_u32(h1[2], s2); o1.w = hmul2_u32(h1[3], s2);
        *reinterpret_cast<uint4*>(tile + sw128_off(r, 2 * b)) = o0;
        *reinterpret_cast<uint4*>(tile + sw128_off(r, 2 * b + 1)) = o1;
    }
}

__device__ __forceinline__ void zero_row(uint8_t* tile, int r) {
#pragma unroll
    for (int c = 0; c < 16; ++c) *reinterpret_cast<uint4*>(tile + sw128_off(r, c)) = make_uint4(0, 0, 0, 0);
}

__global__ void __launch_bounds__(kThreadsTc, 2) attention_tc_kernel(const TcArgs a) {
    extern __shared__ uint8_t smem_raw[];
    __shared__ __align__(8) uint64_t mbar_s;
    __shared__ uint32_t tmem_base_s;
    __shared__ int abort_s;

    const int tid = threadIdx.x;
    const int warp = tid >> 5;
    const int h = blockIdx.y;
    const int m0 = blockIdx.x * kRows;
    const int H = a.H, T_c = a.T_c;

    // 1024-byte aligned operand tiles (the swizzle pattern repeats every 1 KB)
    const uint32_t raw = smem_u32(smem_raw);
    uint8_t* base = smem_raw + (((raw + 1023u) & ~1023u) - raw);
    uint8_t* Qs = base;
    uint8_t* Ks = base + kTileBytes;
    uint8_t* Vs = base + 2 * kTileBytes;
    const uint32_t mbar = smem_u32(&mbar_s);

    if (warp == 0) {
        asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                         smem_u32(&tmem_base_s)),
                     "r"(kTmemCols));
        asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
    }
    if (tid == 0) {
        abort_s = 0;
        asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(mbar), "r"(1));
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }

    // Q row -> fp16 (row scaled by 2^-e into fp16 range), swizzled K-major
    const int qrow = m0 + tid;
    float qexp = 1.0f;                  // 2^e for this row
    {
        uint4 w[16];
        const bool valid = qrow < a.T_q;
        const uint4* src = reinterpret_cast<const uint4*>(a.Q + ((size_t)qrow * H + h) * kHeadDim);
#pragma unroll
        for (int c = 0; c < 16; ++c) w[c] = valid ? src[c] : make_uint4(0, 0, 0, 0);
        uint32_t amax_bits = 0;
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            const uint32_t u[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                amax_bits = max(amax_bits, (u[j] << 16) & 0x7FFFFFFFu);
                amax_bits = max(amax_bits, u[j] & 0x7FFF0000u);
            }
        }
        // exponent e with amax * 2^-e in [2^14, 2^15)
        int e = 0;
        if (amax_bits != 0) e = max(-120, min(120, (int)(amax_bits >> 23) - 127 - 14));
        const float down = __uint_as_float((uint32_t)(127 - e) << 23);   // 2^-e
        qexp = __uint_as_float((uint32_t)(127 + e) << 23);               // 2^e
#pragma unroll
        for (int c = 0; c < 16; ++c) {
            float f[8];
            unpack_bf16x8(w[c], f);
            uint4 o;
            o.x = pack_f16x2(f[0] * down, f[1] * down);
            o.y = pack_f16x2(f[2] * down, f[3] * down);
            o.z = pack_f16x2(f[4] * down, f[5] * down);
            o.w = pack_f16x2(f[6] * down, f[7] * down);
            *reinterpret_cast<uint4*>(Qs + sw128_off(tid, c)) = o;
        }
    }

    // s_Vmax over the key set (every chunk's s_V is positive)
    float sVmax = 0.0f;
    for (int ci = 0; ci < a.n_chunks; ++ci) sVmax = fmaxf(sVmax, a.chunk[ci].tensor_scales[1]);

    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base_s;
    const uint32_t lane_base = (uint32_t)(warp * 32) << 16;
    const uint32_t tS = tmem + lane_base;            // this warp's lanes, S columns
    const uint32_t tO = tmem + lane_base + kOCol;    // this warp's lanes, O columns

    constexpr uint32_t idesc_qk = umma_idesc_f16(false);
    constexpr uint32_t idesc_pv = umma_idesc_f16(true);
    const uint32_t qs_addr = smem_u32(Qs), ks_addr = smem_u32(Ks), vs_addr = smem_u32(Vs);

    float m_run = -INFINITY, l_run = 0.0f;
    uint32_t phase = 0;
    bool o_written = false;
    bool failed = false;

    for (int ci = 0; ci < a.n_chunks && !failed; ++ci) {
        const TcChunk cp = a.chunk[ci];
        const float sK = cp.tensor_scales[0];
        const float rV = cp.tensor_scales[1] / sVmax;
        // Q . mean_c for this row, from the bf16 row
        float qmu = 0.0f;
        if (qrow < a.T_q) {
            const uint4* src = reinterpret_cast<const uint4*>(a.Q + ((size_t)qrow * H + h) * kHeadDim);
            const float4* mp = reinterpret_cast<const float4*>(cp.k_mean + h * kHeadDim);
#pragma unroll 4
            for (int c = 0; c < 16; ++c) {
                float f[8];
                unpack_bf16x8(src[c], f);
                const float4 m0v = mp[2 * c], m1v = mp[2 * c + 1];
                qmu = fmaf(f[0], m0v.x, qmu); qmu = fmaf(f[1], m0v.y, qmu);
                qmu = fmaf(f[2], m0v.z, qmu); qmu = fmaf(f[3], m0v.w, qmu);
                qmu = fmaf(f[4], m1v.x, qmu); qmu = fmaf(f[5], m1v.y, qmu);
                qmu = fmaf(f[6], m1v.z, qmu); qmu = fmaf(f[7], m1v.w, qmu);
            }
        }
        const float alpha = qexp * sK * a.scale_log2;
        const float beta = qmu * a.scale_log2;

        for (int j0 = 0; j0 < T_c; j0 += kKeys) {
            // 1. de-quantize the K and V tiles (thread = key)
            const int key = j0 + tid;
            if (key < T_c) {
                const size_t row = (size_t)h * T_c + key;
                dequant_row(cp.k_codes + row * 64, cp.k_scales + row * 8, Ks, tid);
                dequant_row(cp.v_codes + row * 64, cp.v_scales + row * 8, Vs, tid);
            } else {
                zero_row(Ks, tid);
                zero_row(Vs, tid);
            }
            fence_async_smem();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();

            // 2. S = Q Kq^T
            if (tid == 0) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks) {
                    const uint32_t off = (uint32_t)((ks >> 2) * 16384 + (ks & 3) * 32);
                    mma_ss(tmem, umma_desc(qs_addr + off, 16, 1024),
                           umma_desc(ks_addr + off, 16, 1024), idesc_qk, ks > 0 ? 1u : 0u);
                }
                mma_commit(mbar);
            }
            if (!mbar_wait(mbar, phase)) {
                abort_s = 1;
                record_timeout(a.ctl, 1u, (unsigned)(ci << 16 | (j0 / kKeys)), phase);
            }
            phase ^= 1u;
            __syncthreads();                 // the abort decision is CTA-uniform
            if (abort_s) { failed = true; break; }
            tc_fence_after();

            // 3. softmax on this row
            uint32_t s[128];
            tmem_ld32(tS + 0, s);
            tmem_ld32(tS + 32, s + 32);
            tmem_ld32(tS + 64, s + 64);
            tmem_ld32(tS + 96, s + 96);
            tmem_wait_ld();
            const int valid = min(kKeys, T_c - j0);
            float mx = -INFINITY;
#pragma unroll
            for (int i = 0; i < 128; ++i) {
                const float z = i < valid ? fmaf(__uint_as_float(s[i]), alpha, beta) : -INFINITY;
                s[i] = __float_as_uint(z);
                mx = fmaxf(mx, z);
            }
            // Lazy max: a row moves its reference max (and rescales its O row
            // and sum) only when the new max exceeds it by more than 2^8.  The
            // TMEM loads and stores are warp-collective, so a warp rescales
            // together whenever any of its rows must; the others use factor 1.
            const bool grow = mx > m_run + kRescaleThreshold || m_run == -INFINITY;
            float corr = 1.0f;
            if (grow) {
                const float m_new = fmaxf(mx, m_run);
                corr = ex2f(m_run - m_new);                 // 0 when m_run = -inf
                l_run *= corr;
                m_run = m_new;
            }
            if (o_written && __any_sync(0xFFFFFFFFu, grow)) {
#pragma unroll
                for (int q = 0; q < 4; ++q) {
                    uint32_t ov[32];
                    tmem_ld32(tO + 32 * q, ov);
                    tmem_wait_ld();
#pragma unroll
                    for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * corr);
                    tmem_st32(tO + 32 * q, ov);
                }
            }
            float lsum = 0.0f;
            uint32_t p[64];
#pragma unroll
            for (int i = 0; i < 64; ++i) {
                const float p0 = ex2f(__uint_as_float(s[2 * i]) - m_run);
                const float p1 = ex2f(__uint_as_float(s[2 * i + 1]) - m_run);
                lsum += p0 + p1;
                p[i] = pack_f16x2(p0 * rV, p1 * rV);
            }
            l_run += lsum;
            tmem_st32(tS + 0, p);
            tmem_st32(tS + 32, p + 32);
            tmem_wait_st();
            tc_fence_before();
            __syncthreads();
            tc_fence_after();

            // 4. O += P Vq (P from TMEM columns [0, 64))
            if (tid == 0) {
#pragma unroll
                for (int ks = 0; ks < 8; ++ks)
                    mma_ts(tmem + kOCol, tmem + (uint32_t)(ks * 8),
                           umma_desc(vs_addr + (uint32_t)(ks * 2048), 16384, 1024), idesc_pv,
                           (ks > 0 || o_written) ? 1u : 0u);
                mma_commit(mbar);
            }
            o_written = true;
            if (!mbar_wait(mbar, phase)) {
                abort_s = 1;
                record_timeout(a.ctl, 2u, (unsigned)(ci << 16 | (j0 / kKeys)), phase);
            }
            phase ^= 1u;
            __syncthreads();
            if (abort_s) { failed = true; break; }
            tc_fence_after();
        }
    }

    if (failed) {
        // give the MMAs still in flight a bounded last chance before the
        // tensor memory they write is released
        if (tid == 0) mbar_wait(mbar, phase ^ 1u);
    } else {
        // epilogue: O / l * s_Vmax
        const float inv = sVmax / l_run;
        uint32_t ov[128];
        tmem_ld32(tO + 0, ov);
        tmem_ld32(tO + 32, ov + 32);
        tmem_ld32(tO + 64, ov + 64);
        tmem_ld32(tO + 96, ov + 96);
        tmem_wait_ld();
        if (qrow < a.T_q) {
            const size_t o = ((size_t)qrow * H + h) * kHeadDim;
            if (a.o_f32) {
                float4* dst = reinterpret_cast<float4*>(static_cast<float*>(a.O) + o);
#pragma unroll
                for (int c = 0; c < 32; ++c)
                    dst[c] = make_float4(__uint_as_float(ov[4 * c]) * inv, __uint_as_float(ov[4 * c + 1]) * inv,
                                         __uint_as_float(ov[4 * c + 2]) * inv, __uint_as_float(ov[4 * c + 3]) * inv);
            } else {
                uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(a.O) + o);
#pragma unroll
                for (int c = 0; c < 16; ++c) {
                    uint32_t w[4];
#pragma unroll
                    for (int j = 0; j < 4; ++j) {
                        __nv_bfloat162 b2 = __floats2bfloat162_rn(__uint_as_float(ov[8 * c + 2 * j]) * inv,
                                                                  __uint_as_float(ov[8 * c + 2 * j + 1]) * inv);
                        w[j] = *reinterpret_cast<uint32_t*>(&b2);
                    }
                    dst[c] = make_uint4(w[0], w[1], w[2], w[3]);
                }
            }
        }
    }
    tc_fence_before();
    __syncthreads();
    if (warp == 0) {
        tc_fence_after();
        asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem),
                     "r"(kTmemCols));
    }
}

}  // namespace

nvfp4kv_status launch_attention_tc(const nvfp4kv_chunk_view* chunks, int n_chunks, int T_c,
                                   int H, const void* Q, int T_q, void* O, int o_dtype,
                                   float softmax_scale, void* ws, cudaStream_t stream) {
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(attention_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemTc) != cudaSuccess)
            return NVFP4KV_ERR_CUDA;
        configured = true;
    }
    TcArgs a;
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
    a.Q = static_cast<const uint16_t*>(Q);
    a.O = O;
    a.o_f32 = o_dtype == NVFP4KV_F32 ? 1 : 0;
    a.scale_log2 = softmax_scale * kLog2eTc;
    a.ctl = static_cast<Control*>(ws);
    dim3 grid((T_q + kRows - 1) / kRows, H);
    attention_tc_kernel<<<grid, kThreadsTc, kSmemTc, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

}  // namespace nvfp4kv
