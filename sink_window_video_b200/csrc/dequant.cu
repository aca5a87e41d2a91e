// dequant.cu -- the inverse of the chunk quantizer: NVFP4 codes, E4M3 block
// scales and the FP32 tensor scale (plus K's channel mean) back to fp32 or
// bf16 values in the [T][H][d] token-major layout.
//
// Format: "2605-LongLive2" DeepRead page, Method > 推理基础设施 (NVFP4 KV cache,
// K-smoothing); a decoded element is code value x block scale x tensor scale,
// and K gets its channel mean added back.  Pure streaming work: 0.56 bytes
// read and 2 or 4 bytes written per element, so the kernel is an HBM copy
// with a little arithmetic.
//
// The cache is head-major ([H][T] rows of 64 code bytes and 8 scale bytes)
// and the output token-major, so the kernel moves tiles of kTileTokens
// tokens x up to kTileHeads heads: a persistent CTA prefetches its next tile
// into shared memory with cp.async (one 16-byte copy per quarter code row,
// one 8-byte copy per scale row: every head's rows of the tile are one
// contiguous run in HBM) while it decodes the current one, and every thread
// writes consecutive 16-byte pieces of the output tile (one contiguous run
// when the tile holds all heads) with streaming stores.
#include "common.cuh"
#include "kernels.h"

namespace nvfp4kv {
namespace {

constexpr int kTileTokens = 8;      // even: keeps the second buffer 16-byte aligned
constexpr int kTileHeads = 32;
constexpr int kDequantThreads = 256;
// A buffer holds the tile's codes [token][head][64 B] and scales
// [token][head][8 B] for hb = min(H, kTileHeads) heads; each token's rows
// carry 64 (8) bytes of padding so that both the cp.async writes (8
// consecutive tokens of one head per warp) and the decode reads (16
// consecutive words, then the next head) are free of bank conflicts.
struct TileShape {
    int code_stride, scale_stride, buffer_bytes;
};

inline TileShape tile_shape(int H) {
    const int hb = H < kTileHeads ? H : kTileHeads;
    TileShape s;
    s.code_stride = hb * 64 + 64;
    s.scale_stride = hb * 8 + 8;
    s.buffer_bytes = kTileTokens * (s.code_stride + s.scale_stride);   // a multiple of 16
    return s;
}

constexpr int kMaxDevices = 64;
// CTAs of dequant_kernel resident per SM, per device ordinal and head-block
// width (0 = not yet asked); written by the host before the first launch.
int g_dequant_per_sm[kMaxDevices][kTileHeads];

struct DequantArgs {
    const uint8_t* codes[2];
    const uint8_t* scales[2];
    const float* mean;                  // K's [H][d]
    const float* tensor_scales;         // [s_K, s_V]
    void* out[2];
    int which[2];                       // tensor of each of the n_tensors slots
    int n_tensors, T, H, n_hb, tiles_per_tensor, out_bf16;
    int code_stride, scale_stride, buffer_bytes;
    float one;                          // 1, as a run-time value (see decode8)
};

__device__ __forceinline__ uint32_t smem_addr(const void* p) {
    return (uint32_t)__cvta_generic_to_shared(p);
}

// f16 -> f32 through the mixed-precision add (x + -0 = x for every x, +0
// included): exact, and one full-rate instruction per element.
__device__ __forceinline__ float2 f16x2_to_f32x2_exact(uint32_t h2) {
    float lo, hi;
    asm("{.reg .b16 l, h;\n"
        "mov.b32 {l, h}, %2;\n"
        "add.rn.f32.f16 %0, l, 0f80000000;\n"
        "add.rn.f32.f16 %1, h, 0f80000000;}"
        : "=f"(lo), "=f"(hi)
        : "r"(h2));
    return make_float2(lo, hi);
}

// Eight decoded elements: x = RN(code * D) (+ mean, one more RN), each step
// one IEEE fp32 operation, on float pairs.  The mean is added as
// fma(mean, one, x) with one = 1 held in a run-time value: the same single
// rounding, and a form the compiler cannot merge with the product before it.
__device__ __forceinline__ void decode8(uint32_t q, float D, const float* mean, float one,
                                        float2* x) {
    uint32_t hq[4];
    cvt_e2m1x8_to_f16x2(q, hq);
    const float2 D2 = make_float2(D, D);
#pragma unroll
    for (int j = 0; j < 4; ++j) x[j] = __fmul2_rn(f16x2_to_f32x2_exact(hq[j]), D2);
    if (mean) {
        const float4 m0 = __ldg(reinterpret_cast<const float4*>(mean));
        const float4 m1 = __ldg(reinterpret_cast<const float4*>(mean) + 1);
        const float2 ONE = make_float2(one, one);
        x[0] = __ffma2_rn(make_float2(m0.x, m0.y), ONE, x[0]);
        x[1] = __ffma2_rn(make_float2(m0.z, m0.w), ONE, x[1]);
        x[2] = __ffma2_rn(make_float2(m1.x, m1.y), ONE, x[2]);
        x[3] = __ffma2_rn(make_float2(m1.z, m1.w), ONE, x[3]);
    }
}

struct Tile {
    int w, t0, nt, h0, nh;
};

__device__ __forceinline__ Tile tile_of(const DequantArgs& a, int u) {
    Tile t;
    const int slot = u / a.tiles_per_tensor;
    const int r = u - slot * a.tiles_per_tensor;
    const int tt = r / a.n_hb;
    const int hb = r - tt * a.n_hb;
    t.w = slot == 0 ? a.which[0] : a.which[1];     // selects keep the parameters in constant memory
    t.t0 = tt * kTileTokens;
    t.nt = min(kTileTokens, a.T - t.t0);
    t.h0 = hb * kTileHeads;
    t.nh = min(kTileHeads, a.H - t.h0);
    return t;
}

// Queue the cp.async copies of one tile into buffer buf and close the group.
__device__ __forceinline__ void prefetch_tile(const DequantArgs& a, const Tile& t, uint8_t* buf) {
    uint8_t* cs = buf;
    uint8_t* ss = buf + kTileTokens * a.code_stride;
    const uint8_t* gc = t.w ? a.codes[1] : a.codes[0];
    const uint8_t* gs = t.w ? a.scales[1] : a.scales[0];
    for (int u = threadIdx.x; u < t.nh * kTileTokens * 4; u += kDequantThreads) {
        const int h = u / (kTileTokens * 4);
        const int rem = u - h * kTileTokens * 4;
        const int tt = rem >> 2, qq = rem & 3;
        if (tt < t.nt) {
            const size_t row = (size_t)(t.h0 + h) * a.T + t.t0 + tt;
            asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(
                             smem_addr(cs + tt * a.code_stride + h * 64 + qq * 16)),
                         "l"(gc + row * 64 + qq * 16)
                         : "memory");
        }
    }
    for (int u = threadIdx.x; u < t.nh * kTileTokens; u += kDequantThreads) {
        const int h = u / kTileTokens, tt = u - h * kTileTokens;
        if (tt < t.nt) {
            const size_t row = (size_t)(t.h0 + h) * a.T + t.t0 + tt;
            asm volatile("cp.async.ca.shared.global [%0], [%1], 8;" ::"r"(
                             smem_addr(ss + tt * a.scale_stride + h * 8)),
                         "l"(gs + row * 8)
                         : "memory");
        }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
}

__global__ void __launch_bounds__(kDequantThreads, 6) dequant_kernel(const DequantArgs a) {
    extern __shared__ __align__(16) uint8_t smem[];
    const int units = a.n_tensors * a.tiles_per_tensor;
    int b = 0;
    if ((int)blockIdx.x < units) prefetch_tile(a, tile_of(a, blockIdx.x), smem);
    for (int u = blockIdx.x; u < units; u += gridDim.x) {
        const int nxt = u + gridDim.x;
        if (nxt < units)
            prefetch_tile(a, tile_of(a, nxt), smem + (b ^ 1) * a.buffer_bytes);
        else
            asm volatile("cp.async.commit_group;" ::: "memory");
        asm volatile("cp.async.wait_group 1;" ::: "memory");
        __syncthreads();
        const Tile t = tile_of(a, u);
        const uint8_t* cs = smem + b * a.buffer_bytes;
        const uint8_t* ss = cs + kTileTokens * a.code_stride;
        const float s = a.tensor_scales[t.w];
        void* out = t.w ? a.out[1] : a.out[0];
        const float* mean = t.w == 0 ? a.mean : nullptr;
        // piece c of the tile: token tt = c / (16 nh), head h, 8-channel group g;
        // the stride is a multiple of 16, so g is fixed per thread
        const int n_pieces = t.nt * t.nh * 16;
        const int g = threadIdx.x & 15;
        const int r = threadIdx.x >> 4;
        int tt = r / t.nh, h = r - tt * t.nh;
        // the (token, head) step of one stride: 16 pieces rows further on
        const int dtt = (kDequantThreads / 16) / t.nh;
        const int dh = (kDequantThreads / 16) - dtt * t.nh;
        for (int c = threadIdx.x; c < n_pieces; c += kDequantThreads) {
            const uint32_t q = *reinterpret_cast<const uint32_t*>(cs + tt * a.code_stride + h * 64 + g * 4);
            const float D = __fmul_rn(e4m3_to_f32(ss[tt * a.scale_stride + h * 8 + (g >> 1)]), s);
            float2 x[4];
            decode8(q, D, mean ? mean + (t.h0 + h) * kHeadDim + g * 8 : nullptr, a.one, x);
            const size_t o = ((size_t)(t.t0 + tt) * a.H + t.h0 + h) * kHeadDim + g * 8;
            if (a.out_bf16) {
                uint32_t wv[4];
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                    __nv_bfloat162 p = __floats2bfloat162_rn(x[j].x, x[j].y);
                    wv[j] = *reinterpret_cast<uint32_t*>(&p);
                }
                __stcs(reinterpret_cast<uint4*>(static_cast<uint16_t*>(out) + o),
                       make_uint4(wv[0], wv[1], wv[2], wv[3]));
            } else {
                float4* p = reinterpret_cast<float4*>(static_cast<float*>(out) + o);
                __stcs(p, make_float4(x[0].x, x[0].y, x[1].x, x[1].y));
                __stcs(p + 1, make_float4(x[2].x, x[2].y, x[3].x, x[3].y));
            }
            tt += dtt;
            h += dh;
            if (h >= t.nh) {
                h -= t.nh;
                ++tt;
            }
        }
        __syncthreads();            // buffer b is refilled by the next prefetch
        b ^= 1;
    }
    asm volatile("cp.async.wait_group 0;" ::: "memory");
}

}  // namespace

nvfp4kv_status launch_dequantize(const nvfp4kv_chunk_view& in, int T, int H, void* K_out,
                                 void* V_out, int out_dtype, cudaStream_t stream) {
    if (!K_out && !V_out) return NVFP4KV_OK;
    DequantArgs a;
    a.codes[0] = in.k_codes;
    a.codes[1] = in.v_codes;
    a.scales[0] = in.k_scales;
    a.scales[1] = in.v_scales;
    a.mean = in.k_mean;
    a.tensor_scales = in.tensor_scales;
    a.out[0] = K_out;
    a.out[1] = V_out;
    a.n_tensors = 0;
    if (K_out) a.which[a.n_tensors++] = 0;
    if (V_out) a.which[a.n_tensors++] = 1;
    a.T = T;
    a.H = H;
    a.n_hb = (H + kTileHeads - 1) / kTileHeads;
    a.tiles_per_tensor = ((T + kTileTokens - 1) / kTileTokens) * a.n_hb;
    a.out_bf16 = out_dtype == NVFP4KV_BF16 ? 1 : 0;
    a.one = 1.0f;
    const TileShape ts = tile_shape(H);
    a.code_stride = ts.code_stride;
    a.scale_stride = ts.scale_stride;
    a.buffer_bytes = ts.buffer_bytes;
    const int smem = 2 * ts.buffer_bytes;
    // resident CTAs per SM for this buffer size, asked once per device and size
    // (the buffer size depends on min(H, kTileHeads) only)
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return NVFP4KV_ERR_CUDA;
    const int hb = H < kTileHeads ? H : kTileHeads;
    int& per_sm = g_dequant_per_sm[dev][hb - 1];
    if (per_sm == 0 &&
        (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, dequant_kernel, kDequantThreads,
                                                       smem) != cudaSuccess ||
         per_sm < 1)) {
        per_sm = 0;
        return NVFP4KV_ERR_CUDA;
    }
    const int sms = sm_count_cached();
    if (sms <= 0) return NVFP4KV_ERR_CUDA;
    // as many rounds as the resident CTAs need, then the fewest CTAs that
    // still finish in that many rounds, so that every CTA gets the same count
    const long units = (long)a.n_tensors * a.tiles_per_tensor;
    const long slots = (long)sms * per_sm;
    const long rounds = (units + slots - 1) / slots;
    const int grid = (int)((units + rounds - 1) / rounds);
    dequant_kernel<<<grid, kDequantThreads, smem, stream>>>(a);
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

}  // namespace nvfp4kv
