// quant.cu -- chunk-level NVFP4 quantization of K and V with K-smoothing and
// Four-Over-Six block scales, its inverse, and the format-check kernel.
//
// Method ("2605-LongLive2" DeepRead page, Method > 推理基础设施 and
// 训练基础设施; tailorednewshub page, Inferenza W4A4 NVFP4): per chunk and per
// tensor, an FP32 tensor scale s = max|X| / (6*448); per 16-channel block an
// E4M3 scale and sixteen E2M1 codes, the block max mapped to 6 and to 4, the
// lower squared error kept; K has its per-head, per-channel mean over the
// chunk's tokens removed first and kept in fp32.
//
// One cooperative persistent kernel per chunk, three phases split by grid
// barriers:
//   1. stats:    every (64-token segment, 256-column group) of K gives column
//                sums (fp32, in token order), column min and max (bf16, exact);
//                V gives per-CTA max |V|.  One 128-bit load per lane per token.
//   2. finalize: per column, the segment sums are added in segment order and
//                divided by T (the mean); max |K - mean| comes from the column
//                min/max (x -> RN(x - mean) is monotone), reduced per CTA.
//   3. encode:   two lanes per 16-element block (8 elements each, one 128-bit
//                load); the block max and the two half-errors meet through one
//                shuffle each; each lane of a pair computes one target's block
//                scale and swaps it with its partner; codes are stored packed,
//                head-major, 4 bytes per lane.
// Every fp32 step that the definition fixes is one IEEE operation (explicit
// _rn intrinsics, compiled without FMA contraction), so codes, scales, means
// and tensor scales are bit-identical to the definition.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4kv {
namespace {

constexpr int kQuantThreads = 256;
constexpr int kQuantWarps = kQuantThreads / 32;

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

// ---------------------------------------------------------------- phase 1

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

__device__ __forceinline__ void stats_v_token(const uint4& w, uint32_t* mx) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) mx[j] = as_u32(__hmax2(as_bf162(mx[j]), as_bf162(u[j] & 0x7FFF7FFFu)));
}

__device__ void phase_stats(const QuantArgs& a, float* red) {
    const int lane = threadIdx.x & 31;
    const int wg = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
    const int nw = gridDim.x * kQuantWarps;
    const int upt = a.nseg * a.ngroups;
    const size_t row8 = (size_t)a.HD / 8;
    float vmax = 0.0f;
    for (int u = wg; u < 2 * upt; u += nw) {
        const bool isK = u < upt;
        const int uu = isK ? u : u - upt;
        const int s = uu / a.ngroups;
        const int g = uu - s * a.ngroups;
        const int col = g * 256 + lane * 8;
        if (col >= a.HD) continue;
        const int t0 = s * kSegment;
        const int nt = min(kSegment, a.T - t0);
        const uint4* src = (isK ? a.K : a.V) + (size_t)t0 * row8 + col / 8;
        if (isK) {
            float sum[8];
            uint32_t mn[4], mx[4];
#pragma unroll
            for (int i = 0; i < 8; ++i) sum[i] = 0.0f;
#pragma unroll
            for (int j = 0; j < 4; ++j) { mn[j] = 0x7F807F80u; mx[j] = 0xFF80FF80u; }
            int t = 0;
            for (; t + 8 <= nt; t += 8) {
                uint4 w[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) w[k] = ld_stream(src + (size_t)(t + k) * row8);
#pragma unroll
                for (int k = 0; k < 8; ++k) stats_k_token(w[k], sum, mn, mx);
            }
            for (; t < nt; ++t) stats_k_token(ld_stream(src + (size_t)t * row8), sum, mn, mx);
            float4* ps = reinterpret_cast<float4*>(a.psum + (size_t)s * a.HD + col);
            ps[0] = make_float4(sum[0], sum[1], sum[2], sum[3]);
            ps[1] = make_float4(sum[4], sum[5], sum[6], sum[7]);
            const size_t w2 = ((size_t)s * a.HD + col) / 2;
            *reinterpret_cast<uint4*>(a.pmin + w2) = make_uint4(mn[0], mn[1], mn[2], mn[3]);
            *reinterpret_cast<uint4*>(a.pmax + w2) = make_uint4(mx[0], mx[1], mx[2], mx[3]);
        } else {
            uint32_t mx[4] = {0u, 0u, 0u, 0u};
            int t = 0;
            for (; t + 8 <= nt; t += 8) {
                uint4 w[8];
#pragma unroll
                for (int k = 0; k < 8; ++k) w[k] = ld_stream(src + (size_t)(t + k) * row8);
#pragma unroll
                for (int k = 0; k < 8; ++k) stats_v_token(w[k], mx);
            }
            for (; t < nt; ++t) stats_v_token(ld_stream(src + (size_t)t * row8), mx);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
                vmax = fmaxf(vmax, __uint_as_float(mx[j] << 16));
                vmax = fmaxf(vmax, __uint_as_float(mx[j] & 0xFFFF0000u));
            }
        }
    }
    const float b = block_max(vmax, red);
    if (threadIdx.x == 0) a.vpart[blockIdx.x] = b;
}

// ---------------------------------------------------------------- phase 2

__device__ void phase_finalize(const QuantArgs& a, float* red) {
    float kp = 0.0f;
    const int stride = gridDim.x * blockDim.x;
    const float Tf = (float)a.T;
    const unsigned short* pmin = reinterpret_cast<const unsigned short*>(a.pmin);
    const unsigned short* pmax = reinterpret_cast<const unsigned short*>(a.pmax);
    for (int col = blockIdx.x * blockDim.x + threadIdx.x; col < a.HD; col += stride) {
        float S = 0.0f, mn = INFINITY, mx = -INFINITY;
        int s = 0;
        for (; s + 8 <= a.nseg; s += 8) {
            float p[8];
            unsigned short n[8], x[8];
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                const size_t i = (size_t)(s + k) * a.HD + col;
                p[k] = __ldcg(a.psum + i);
                n[k] = __ldcg(pmin + i);
                x[k] = __ldcg(pmax + i);
            }
#pragma unroll
            for (int k = 0; k < 8; ++k) {
                S = __fadd_rn(S, p[k]);
                mn = fminf(mn, __uint_as_float((uint32_t)n[k] << 16));
                mx = fmaxf(mx, __uint_as_float((uint32_t)x[k] << 16));
            }
        }
        for (; s < a.nseg; ++s) {
            const size_t i = (size_t)s * a.HD + col;
            S = __fadd_rn(S, __ldcg(a.psum + i));
            mn = fminf(mn, __uint_as_float((uint32_t)__ldcg(pmin + i) << 16));
            mx = fmaxf(mx, __uint_as_float((uint32_t)__ldcg(pmax + i) << 16));
        }
        const float mu = __fdiv_rn(S, Tf);
        a.k_mean[col] = mu;
        kp = fmaxf(kp, fmaxf(fabsf(__fsub_rn(mx, mu)), fabsf(__fsub_rn(mn, mu))));
    }
    const float b = block_max(kp, red);
    if (threadIdx.x == 0) a.kpart[blockIdx.x] = b;
}

// ---------------------------------------------------------------- phase 3

// Eight elements x against one candidate (block step D, its reciprocal r):
// packed codes q (byte j = elements 2j, 2j+1) and the sequential sum of the
// eight squared errors (x - decode(q) * D)^2.
__device__ __forceinline__ void encode_half(const float* x, float D, float r, uint32_t& q,
                                            float& err) {
    float y[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) y[i] = div_markstein(x[i], D, r);
    q = D > 0.0f ? cvt_e2m1x8(y) : 0u;
    uint32_t h[4];
    cvt_e2m1x8_to_f16x2(q, h);
    float acc = 0.0f;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        const float e0 = __fsub_rn(x[2 * j], __fmul_rn(f16lo(h[j]), D));
        const float e1 = __fsub_rn(x[2 * j + 1], __fmul_rn(f16hi(h[j]), D));
        const float s0 = __fmul_rn(e0, e0);
        const float s1 = __fmul_rn(e1, e1);
        acc = (j == 0) ? s0 : __fadd_rn(acc, s0);
        acc = __fadd_rn(acc, s1);
    }
    err = acc;
}

__device__ void phase_encode(const QuantArgs& a, float* red) {
    float kp = 0.0f, vp = 0.0f;
    for (int i = threadIdx.x; i < gridDim.x; i += blockDim.x) {
        kp = fmaxf(kp, __ldcg(a.kpart + i));
        vp = fmaxf(vp, __ldcg(a.vpart + i));
    }
    const float AK = block_max(kp, red);
    const float AV = block_max(vp, red);
    const float sK = AK > 0.0f ? __fdiv_rn(AK, kTensorScaleDiv) : 1.0f;
    const float sV = AV > 0.0f ? __fdiv_rn(AV, kTensorScaleDiv) : 1.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) {
        a.tensor_scales[0] = sK;
        a.tensor_scales[1] = sV;
    }

    const int lane = threadIdx.x & 31;
    const int wg = blockIdx.x * kQuantWarps + (threadIdx.x >> 5);
    const int nw = gridDim.x * kQuantWarps;
    const int tiles = (a.T + 15) / 16;
    const int upt = a.H * tiles;
    const int c8 = lane & 15;                 // 8-channel group of this lane
    const bool odd = (lane & 1) != 0;         // second half of its 16-block
    for (int u = wg; u < 2 * upt; u += nw) {
        const bool isK = u < upt;
        const int uu = isK ? u : u - upt;
        const int h = uu / tiles;
        const int tile = uu - h * tiles;
        const float s = isK ? sK : sV;
        // this lane's target: 6 on the even lane of a pair, 4 on the odd one
        const float ms = __fmul_rn(odd ? 4.0f : 6.0f, s);
        float mu[8];
        if (isK) {
            const float4* mp = reinterpret_cast<const float4*>(a.k_mean + h * kHeadDim + c8 * 8);
            const float4 m0 = __ldcg(mp), m1 = __ldcg(mp + 1);
            mu[0] = m0.x; mu[1] = m0.y; mu[2] = m0.z; mu[3] = m0.w;
            mu[4] = m1.x; mu[5] = m1.y; mu[6] = m1.z; mu[7] = m1.w;
        }
        const uint4* src = isK ? a.K : a.V;
        uint32_t* codes = reinterpret_cast<uint32_t*>(isK ? a.k_codes : a.v_codes);
        uint8_t* scales = isK ? a.k_scales : a.v_scales;
#pragma unroll 2
        for (int it = 0; it < 8; ++it) {
            const int t = tile * 16 + it * 2 + (lane >> 4);
            const bool valid = t < a.T;
            const uint4 w = valid ? ld_stream(src + ((size_t)t * a.H + h) * 16 + c8)
                                  : make_uint4(0u, 0u, 0u, 0u);
            float x[8];
            unpack_bf16x8(w, x);
            if (isK) {
#pragma unroll
                for (int i = 0; i < 8; ++i) x[i] = __fsub_rn(x[i], mu[i]);
            }
            float ah = 0.0f;
#pragma unroll
            for (int i = 0; i < 8; ++i) ah = fmaxf(ah, fabsf(x[i]));
            const float ab = fmaxf(ah, __shfl_xor_sync(0xFFFFFFFFu, ah, 1));
            // block scale for this lane's target, then swap with the partner
            const float ratio = __fdiv_rn(ab, ms);
            const uint32_t sb = cvt_e4m3x2(ratio, 0.0f) & 0xFFu;
            const float D = __fmul_rn(e4m3_to_f32(sb), s);
            const float r = D > 0.0f ? __frcp_rn(D) : 0.0f;
            const float Do = __shfl_xor_sync(0xFFFFFFFFu, D, 1);
            const float ro = __shfl_xor_sync(0xFFFFFFFFu, r, 1);
            const uint32_t sbo = __shfl_xor_sync(0xFFFFFFFFu, sb, 1);
            const float D6 = odd ? Do : D, r6 = odd ? ro : r;
            const float D4 = odd ? D : Do, r4 = odd ? r : ro;
            const uint32_t sb6 = odd ? sbo : sb, sb4 = odd ? sb : sbo;
            uint32_t q6, q4;
            float e6, e4;
            encode_half(x, D6, r6, q6, e6);
            encode_half(x, D4, r4, q4, e4);
            // block error = (elements 0..7) + (elements 8..15)
            const float E6 = __fadd_rn(e6, __shfl_xor_sync(0xFFFFFFFFu, e6, 1));
            const float E4 = __fadd_rn(e4, __shfl_xor_sync(0xFFFFFFFFu, e4, 1));
            const bool keep4 = E4 < E6;
            if (valid) {
                const size_t row = (size_t)h * a.T + t;
                codes[row * 16 + c8] = keep4 ? q4 : q6;
                if (!odd) scales[row * 8 + (c8 >> 1)] = (uint8_t)(keep4 ? sb4 : sb6);
            }
        }
    }
}

__global__ void __launch_bounds__(kQuantThreads, 2) quantize_kernel(QuantArgs a) {
    __shared__ float red[kQuantWarps];
    phase_stats(a, red);
    if (!grid_barrier(a.ctl)) return;
    phase_finalize(a, red);
    if (!grid_barrier(a.ctl)) return;
    phase_encode(a, red);
}

// ---------------------------------------------------------------- dequantize

// One thread per (head, token, 8-channel group): x = decode(q) * (decode(sb) * s)
// (+ mean for K); output [T][H][d] fp32 or bf16 (nearest even).
__global__ void dequant_kernel(const uint8_t* codes, const uint8_t* scales, const float* mean,
                               const float* tensor_scales, int which, int T, int H, void* out,
                               int out_bf16) {
    const size_t idx = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    const size_t total = (size_t)H * T * 16;
    if (idx >= total) return;
    const int g = (int)(idx & 15);
    const size_t row = idx >> 4;                   // h * T + t
    const int h = (int)(row / T);
    const int t = (int)(row - (size_t)h * T);
    const float s = tensor_scales[which];
    const uint32_t q = reinterpret_cast<const uint32_t*>(codes)[row * 16 + g];
    const float D = __fmul_rn(e4m3_to_f32(scales[row * 8 + (g >> 1)]), s);
    uint32_t hq[4];
    cvt_e2m1x8_to_f16x2(q, hq);
    float x[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
        x[2 * j] = __fmul_rn(f16lo(hq[j]), D);
        x[2 * j + 1] = __fmul_rn(f16hi(hq[j]), D);
    }
    if (mean) {
#pragma unroll
        for (int i = 0; i < 8; ++i) x[i] = __fadd_rn(x[i], mean[h * kHeadDim + g * 8 + i]);
    }
    const size_t o = ((size_t)t * H + h) * kHeadDim + g * 8;
    if (out_bf16) {
        uint32_t w[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
            __nv_bfloat162 p = __floats2bfloat162_rn(x[2 * j], x[2 * j + 1]);
            w[j] = *reinterpret_cast<uint32_t*>(&p);
        }
        *reinterpret_cast<uint4*>(reinterpret_cast<uint16_t*>(out) + o) =
            make_uint4(w[0], w[1], w[2], w[3]);
    } else {
        float4* p = reinterpret_cast<float4*>(reinterpret_cast<float*>(out) + o);
        p[0] = make_float4(x[0], x[1], x[2], x[3]);
        p[1] = make_float4(x[4], x[5], x[6], x[7]);
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
    void* args[] = {&a};
    cudaError_t e = cudaLaunchCooperativeKernel((const void*)quantize_kernel,
                                                dim3(g_quant_grid[dev]), dim3(kQuantThreads),
                                                args, 0, stream);
    return e == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

nvfp4kv_status launch_dequantize(const nvfp4kv_chunk_view& in, int T, int H, void* K_out,
                                 void* V_out, int out_dtype, cudaStream_t stream) {
    const size_t total = (size_t)H * T * 16;
    const int threads = 256;
    const unsigned blocks = (unsigned)((total + threads - 1) / threads);
    if (K_out)
        dequant_kernel<<<blocks, threads, 0, stream>>>(in.k_codes, in.k_scales, in.k_mean,
                                                       in.tensor_scales, 0, T, H, K_out,
                                                       out_dtype);
    if (V_out)
        dequant_kernel<<<blocks, threads, 0, stream>>>(in.v_codes, in.v_scales, nullptr,
                                                       in.tensor_scales, 1, T, H, V_out,
                                                       out_dtype);
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
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
    if (!K || !V || !out || T_c <= 0 || H <= 0 || T_c > (1 << 24) || H > 4096 ||
        !out->k_codes || !out->k_scales || !out->v_codes || !out->v_scales || !out->k_mean ||
        !out->tensor_scales)
        return NVFP4KV_ERR_INVALID_ARG;
    if (d != kHeadDim) return NVFP4KV_ERR_UNSUPPORTED;
    const uintptr_t mis = reinterpret_cast<uintptr_t>(K) | reinterpret_cast<uintptr_t>(V) |
                          reinterpret_cast<uintptr_t>(out->k_codes) |
                          reinterpret_cast<uintptr_t>(out->v_codes) |
                          reinterpret_cast<uintptr_t>(out->k_scales) |
                          reinterpret_cast<uintptr_t>(out->v_scales) |
                          reinterpret_cast<uintptr_t>(out->k_mean);
    if ((mis & 15u) != 0 || (reinterpret_cast<uintptr_t>(out->tensor_scales) & 7u) != 0)
        return NVFP4KV_ERR_ALIGNMENT;
    // the chunk's scratch must fit the compiled-in array
    if (ws_layout(T_c, H).total > kStaticScratchBytes) return NVFP4KV_ERR_CAPACITY;

    int dev = 0, major = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4KV_ERR_CUDA;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess)
        return NVFP4KV_ERR_CUDA;
    if (major != 10) return NVFP4KV_ERR_UNSUPPORTED;
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
    if (cudaMemsetAsync(scratch, 0, sizeof(Control), (cudaStream_t)stream) != cudaSuccess)
        return NVFP4KV_ERR_CUDA;
    return launch_quantize(K, V, T_c, H, *out, scratch, (cudaStream_t)stream);
}
