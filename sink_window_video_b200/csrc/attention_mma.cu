// attention_mma.cu -- sink-window attention over the NVFP4 cache with fused
// de-quantization, on the warp-level tensor-core path (mma.sync m16n8k16,
// bf16 in, fp32 accumulate).  It is the first, plain tensor-core version;
// the tcgen05/TMEM kernel supersedes it on sm_100a, and the two are kept
// cross-checkable.
//
// Method ("2605-LongLive2" DeepRead page, Method > 算法层设计: attention over
// K_eff = A_g u A_s u KV[t-W, t); Method > 推理基础设施: the NVFP4 cache is
// de-quantized inside the attention kernel):
//   K_hat = decode(q) * decode(sb) * s_K + mean,   V_hat = decode(q) * decode(sb) * s_V.
// The product decode(q) * decode(sb) (an E2M1 value times an E4M3 value, at
// most 6 significant bits, magnitude in [2^-10, 2688]) is exact in bf16, so
// the tensor-core operands are the exact cache values; the per-chunk factors
// are applied in fp32 outside the products:
//   Q K_hat^T = s_K (Q Kq^T) + (Q . mean)        (a per-row, per-chunk bias)
//   P V_hat   = (P s_V) Vq
// with Kq, Vq the exact bf16 de-quantized codes.  Online softmax in fp32
// (base-2 exponent), one pass over the key chunks.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4kv {
namespace {

constexpr int kM = 64;              // query rows per CTA (16 per warp)
constexpr int kN = 64;              // keys per tile
constexpr int kThreads = 128;
constexpr int kStride = kHeadDim + 8;   // smem row pitch (bf16), conflict-free ldmatrix
constexpr float kLog2e = 1.4426950408889634f;

struct ChunkPtrs {
    const uint8_t* k_codes;
    const uint8_t* k_scales;
    const uint8_t* v_codes;
    const uint8_t* v_scales;
    const float* k_mean;
    const float* tensor_scales;
};

struct AttnArgs {
    ChunkPtrs chunk[NVFP4KV_MAX_KEY_CHUNKS];
    int n_chunks, T_c, H, T_q;
    const uint16_t* Q;
    void* O;
    int o_f32;                      // 1: float32 output, 0: bf16
    float scale_log2;               // softmax scale * log2(e)
};

__device__ __forceinline__ float ex2(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                        uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2,
                                          uint32_t& r3) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                 : "r"(addr));
}

__device__ __forceinline__ void mma_bf16(float* c, const uint32_t* a, uint32_t b0, uint32_t b1) {
    asm volatile(
        "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, "
        "{%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
        : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
        : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
    __nv_bfloat162 p = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t*>(&p);
}

// De-quantize 64 consecutive codes (32 bytes) with their four block scales
// into 64 bf16 values (exact) at dst.
__device__ __forceinline__ void dequant64(const uint8_t* codes, const uint8_t* scales,
                                          uint16_t* dst) {
    const uint4 c0 = *reinterpret_cast<const uint4*>(codes);
    const uint4 c1 = *reinterpret_cast<const uint4*>(codes + 16);
    const uint32_t sc = *reinterpret_cast<const uint32_t*>(scales);
    const uint32_t cw[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
    const uint32_t s01 = cvt_e4m3x2_to_f16x2(sc & 0xFFFFu);
    const uint32_t s23 = cvt_e4m3x2_to_f16x2(sc >> 16);
    const float sb[4] = {f16lo(s01), f16hi(s01), f16lo(s23), f16hi(s23)};
#pragma unroll
    for (int w = 0; w < 8; ++w) {           // 8 codes per word, block = w / 2
        uint32_t h[4];
        cvt_e2m1x8_to_f16x2(cw[w], h);
        const float b = sb[w >> 1];
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) o[j] = pack_bf16(f16lo(h[j]) * b, f16hi(h[j]) * b);
        *reinterpret_cast<uint4*>(dst + 8 * w) = make_uint4(o[0], o[1], o[2], o[3]);
    }
}

__global__ void __launch_bounds__(kThreads) attention_mma_kernel(const AttnArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    uint16_t* Qs = reinterpret_cast<uint16_t*>(smem);
    uint16_t* Ks = Qs + kM * kStride;
    uint16_t* Vs = Ks + kN * kStride;
    float* mu_s = reinterpret_cast<float*>(Vs + kN * kStride);
    float* qmu_s = mu_s + kHeadDim;

    const int tid = threadIdx.x;
    const int warp = tid >> 5, lane = tid & 31;
    const int g = lane >> 2, tq = lane & 3;
    const int h = blockIdx.y;
    const int m0 = blockIdx.x * kM;
    const int H = a.H, T_c = a.T_c;

    // Q tile -> smem (rows past T_q are zero)
    for (int i = tid; i < kM * 16; i += kThreads) {
        const int r = i >> 4, c = (i & 15) * 8;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (m0 + r < a.T_q)
            v = *reinterpret_cast<const uint4*>(a.Q + ((size_t)(m0 + r) * H + h) * kHeadDim + c);
        *reinterpret_cast<uint4*>(Qs + r * kStride + c) = v;
    }
    __syncthreads();
    uint32_t qa[8][4];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
        const int row = warp * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
        const int col = k * 16 + 8 * (lane >> 4);
        ldsm_x4(smem_addr(Qs + row * kStride + col), qa[k][0], qa[k][1], qa[k][2], qa[k][3]);
    }

    float o[16][4];
#pragma unroll
    for (int n = 0; n < 16; ++n) o[n][0] = o[n][1] = o[n][2] = o[n][3] = 0.0f;
    float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.0f, 0.0f};

    for (int ci = 0; ci < a.n_chunks; ++ci) {
        const ChunkPtrs cp = a.chunk[ci];
        const float sK = cp.tensor_scales[0], sV = cp.tensor_scales[1];
        mu_s[tid] = cp.k_mean[h * kHeadDim + tid];
        __syncthreads();
        {   // Q . mean for the 64 rows: two threads per row
            const int r = tid >> 1, half = tid & 1;
            float acc = 0.0f;
#pragma unroll 8
            for (int c = 0; c < 64; ++c) {
                const int cc = half * 64 + c;
                acc = fmaf(__uint_as_float((uint32_t)Qs[r * kStride + cc] << 16), mu_s[cc], acc);
            }
            acc += __shfl_xor_sync(0xFFFFFFFFu, acc, 1);
            if (half == 0) qmu_s[r] = acc;
        }
        __syncthreads();
        const float alpha = sK * a.scale_log2;
        const float beta0 = qmu_s[warp * 16 + g] * a.scale_log2;
        const float beta1 = qmu_s[warp * 16 + g + 8] * a.scale_log2;

        for (int j0 = 0; j0 < T_c; j0 += kN) {
            {   // de-quantize the K and V tiles: two threads per key, 64 channels each
                const int key = tid >> 1, half = tid & 1;
                uint16_t* kd = Ks + key * kStride + half * 64;
                uint16_t* vd = Vs + key * kStride + half * 64;
                if (j0 + key < T_c) {
                    const size_t row = (size_t)h * T_c + j0 + key;
                    dequant64(cp.k_codes + row * 64 + half * 32, cp.k_scales + row * 8 + half * 4, kd);
                    dequant64(cp.v_codes + row * 64 + half * 32, cp.v_scales + row * 8 + half * 4, vd);
                } else {
#pragma unroll
                    for (int w = 0; w < 8; ++w) {
                        *reinterpret_cast<uint4*>(kd + 8 * w) = make_uint4(0u, 0u, 0u, 0u);
                        *reinterpret_cast<uint4*>(vd + 8 * w) = make_uint4(0u, 0u, 0u, 0u);
                    }
                }
            }
            __syncthreads();

            // S = Q Kq^T : 16 x 64 per warp
            float s[8][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) s[n][0] = s[n][1] = s[n][2] = s[n][3] = 0.0f;
#pragma unroll
            for (int k = 0; k < 8; ++k) {
#pragma unroll
                for (int n = 0; n < 8; n += 2) {
                    const int key = n * 8 + (lane & 7) + 8 * (lane >> 4);
                    const int col = k * 16 + 8 * ((lane >> 3) & 1);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4(smem_addr(Ks + key * kStride + col), b0, b1, b2, b3);
                    mma_bf16(s[n], qa[k], b0, b1);
                    mma_bf16(s[n + 1], qa[k], b2, b3);
                }
            }
            // logits (base 2), masking keys past the chunk's end
            float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
            for (int n = 0; n < 8; ++n) {
#pragma unroll
                for (int e = 0; e < 2; ++e) {
                    const bool ok = j0 + n * 8 + 2 * tq + e < T_c;
                    s[n][e] = ok ? fmaf(s[n][e], alpha, beta0) : -INFINITY;
                    s[n][2 + e] = ok ? fmaf(s[n][2 + e], alpha, beta1) : -INFINITY;
                    mx0 = fmaxf(mx0, s[n][e]);
                    mx1 = fmaxf(mx1, s[n][2 + e]);
                }
            }
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 1));
            mx0 = fmaxf(mx0, __shfl_xor_sync(0xFFFFFFFFu, mx0, 2));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 1));
            mx1 = fmaxf(mx1, __shfl_xor_sync(0xFFFFFFFFu, mx1, 2));
            const float mn0 = fmaxf(mrow[0], mx0), mn1 = fmaxf(mrow[1], mx1);
            const float c0 = ex2(mrow[0] - mn0), c1 = ex2(mrow[1] - mn1);
            mrow[0] = mn0;
            mrow[1] = mn1;
            lrow[0] *= c0;
            lrow[1] *= c1;
#pragma unroll
            for (int n = 0; n < 16; ++n) {
                o[n][0] *= c0; o[n][1] *= c0;
                o[n][2] *= c1; o[n][3] *= c1;
            }
            // P = exp2(logit - max); row sums in fp32; P * s_V in bf16 as A fragments
            uint32_t pa[4][4];
#pragma unroll
            for (int n = 0; n < 8; ++n) {
                const float p0 = ex2(s[n][0] - mn0), p1 = ex2(s[n][1] - mn0);
                const float p2 = ex2(s[n][2] - mn1), p3 = ex2(s[n][3] - mn1);
                lrow[0] += p0 + p1;
                lrow[1] += p2 + p3;
                const int kk = n >> 1, hi = n & 1;
                pa[kk][hi * 2 + 0] = pack_bf16(p0 * sV, p1 * sV);
                pa[kk][hi * 2 + 1] = pack_bf16(p2 * sV, p3 * sV);
            }
            // O += P Vq
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
#pragma unroll
                for (int n = 0; n < 16; n += 2) {
                    const int key = kk * 16 + (lane & 7) + 8 * ((lane >> 3) & 1);
                    const int col = n * 8 + 8 * (lane >> 4);
                    uint32_t b0, b1, b2, b3;
                    ldsm_x4_t(smem_addr(Vs + key * kStride + col), b0, b1, b2, b3);
                    mma_bf16(o[n], pa[kk], b0, b1);
                    mma_bf16(o[n + 1], pa[kk], b2, b3);
                }
            }
            __syncthreads();
        }
    }

    // epilogue: O / l -> bf16
    float l0 = lrow[0], l1 = lrow[1];
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 1);
    l0 += __shfl_xor_sync(0xFFFFFFFFu, l0, 2);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 1);
    l1 += __shfl_xor_sync(0xFFFFFFFFu, l1, 2);
    const float i0 = 1.0f / l0, i1 = 1.0f / l1;
    const int r0 = m0 + warp * 16 + g, r1 = r0 + 8;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
        const int col = n * 8 + 2 * tq;
        const size_t e0 = ((size_t)r0 * H + h) * kHeadDim + col;
        const size_t e1 = ((size_t)r1 * H + h) * kHeadDim + col;
        if (a.o_f32) {
            float* Of = static_cast<float*>(a.O);
            if (r0 < a.T_q) *reinterpret_cast<float2*>(Of + e0) = make_float2(o[n][0] * i0, o[n][1] * i0);
            if (r1 < a.T_q) *reinterpret_cast<float2*>(Of + e1) = make_float2(o[n][2] * i1, o[n][3] * i1);
        } else {
            uint16_t* Ob = static_cast<uint16_t*>(a.O);
            if (r0 < a.T_q) *reinterpret_cast<uint32_t*>(Ob + e0) = pack_bf16(o[n][0] * i0, o[n][1] * i0);
            if (r1 < a.T_q) *reinterpret_cast<uint32_t*>(Ob + e1) = pack_bf16(o[n][2] * i1, o[n][3] * i1);
        }
    }
}

constexpr size_t kSmemBytes =
    (size_t)(kM + 2 * kN) * kStride * 2 + kHeadDim * 4 + kM * 4;

}  // namespace

nvfp4kv_status launch_attention_mma(const nvfp4kv_chunk_view* chunks, int n_chunks, int T_c,
                                    int H, const void* Q, int T_q, void* O, int o_dtype,
                                    float softmax_scale, cudaStream_t stream) {
    static bool configured = false;
    if (!configured) {
        if (cudaFuncSetAttribute(attention_mma_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kSmemBytes) != cudaSuccess)
            return NVFP4KV_ERR_CUDA;
        configured = true;
    }
    AttnArgs a;
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
    a.scale_log2 = softmax_scale * kLog2e;
    dim3 grid((T_q + kM - 1) / kM, H);
    attention_mma_kernel<<<grid, kThreads, kSmemBytes, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}



}  // namespace nvfp4kv
