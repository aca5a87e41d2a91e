// matrix_quant.cu -- NVFP4 quantization of weight and activation matrices with
// Four-Over-Six (DeepRead page, Method > 训练基础设施: NVFP4 weights and
// activations, E2M1 values under FP8 E4M3 block scales and an FP32 tensor
// scale, each block's scale searched over targets 6 and 4).  Activations take
// 16-element blocks along a row, weights 16 x 16 tiles (one scale per tile;
// the tile's error adds its rows' (first 8 + last 8) squared errors in row
// order).
//
// One cooperative persistent kernel, two phases split by a grid barrier:
//   A. max |X|: one streaming pass (L2 evict_last), per-CTA partial maxima;
//   B. the encoding, X re-read from L2 (evict_first): 1D -- 32 consecutive
//      blocks per warp, one lane per block; 2D -- one warp per tile,
//      lane = (row, half row).
// The block arithmetic is the KV quantizer's (nvfp4_encode.cuh), bit-identical
// to the definition.
#include "common.cuh"
#include "kernels.h"
#include "nvfp4_encode.cuh"

namespace nvfp4kv {
namespace {

constexpr int kMqThreads = 768;           // one CTA per SM: 24 warps
constexpr int kMqWarps = kMqThreads / 32;

struct MatArgs {
    const uint4* X;          // [M][N] bf16
    int M, N, mode;          // mode 1: row blocks, 2: 16 x 16 tiles
    uint32_t* codes;         // [M][N/2] bytes, as 32-bit words
    uint8_t* scales;         // [M][N/16] or [M/16][N/16]
    float* tensor_scale;
    float* part;             // per-CTA max |X|
    Control* ctl;
    float one;               // 1 as a run-time value (see encode8_fast)
};

struct MatShared {
    float red[kMqWarps];
    float2 tab[256];         // per E4M3 code: D = RN(code * s), RN(1/D)
};

__device__ __forceinline__ float cta_max(float v, float* red) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
    if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
    __syncthreads();
    float r = red[0];
#pragma unroll
    for (int i = 1; i < kMqWarps; ++i) r = fmaxf(r, red[i]);
    __syncthreads();
    return r;
}

__device__ void phase_amax(const MatArgs& a, MatShared& sh, uint64_t keep) {
    const size_t n16 = (size_t)a.M * a.N / 8;
    const size_t stride = (size_t)gridDim.x * blockDim.x;
    size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x;
    uint32_t m = 0;                               // two bf16 magnitudes, lane-wise max
    for (; i + 15 * stride < n16; i += 16 * stride) {
        uint4 w[16];
#pragma unroll
        for (int k = 0; k < 16; ++k) w[k] = ld_hint(a.X + i + k * stride, keep);
#pragma unroll
        for (int k = 0; k < 16; ++k) {
            m = __vmaxu2(m, w[k].x & 0x7FFF7FFFu);
            m = __vmaxu2(m, w[k].y & 0x7FFF7FFFu);
            m = __vmaxu2(m, w[k].z & 0x7FFF7FFFu);
            m = __vmaxu2(m, w[k].w & 0x7FFF7FFFu);
        }
    }
    for (; i < n16; i += stride) {
        const uint4 w = ld_hint(a.X + i, keep);
        m = __vmaxu2(m, w.x & 0x7FFF7FFFu);
        m = __vmaxu2(m, w.y & 0x7FFF7FFFu);
        m = __vmaxu2(m, w.z & 0x7FFF7FFFu);
        m = __vmaxu2(m, w.w & 0x7FFF7FFFu);
    }
    const float v = fmaxf(__uint_as_float(m << 16), __uint_as_float(m & 0xFFFF0000u));
    const float b = cta_max(v, sh.red);
    if (threadIdx.x == 0) a.part[blockIdx.x] = b;
}

// Both targets of one lane's 8 elements: block scales from the block max ab,
// codes and the lane's half-errors.
struct LaneEnc {
    uint32_t q6, q4, sb6, sb4;
    float e6, e4, D6, D4;
};

__device__ __forceinline__ LaneEnc encode_lane(const float2* x, float ab, const MatShared& sh,
                                               const EncodeConsts& c, float one) {
    LaneEnc r;
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
    r.sb6 = sbp & 0xFFu;
    r.sb4 = sbp >> 8;
    const float2 t6 = sh.tab[r.sb6], t4 = sh.tab[r.sb4];
    r.D6 = t6.x;
    r.D4 = t4.x;
    if (c.fast) {
        encode8_fast(x, t6, one, r.q6, r.e6);
        encode8_fast(x, t4, one, r.q4, r.e4);
    } else {
        const Enc8 a6 = encode8_slow(x[0].x, x[0].y, x[1].x, x[1].y, x[2].x, x[2].y, x[3].x,
                                     x[3].y, t6.x);
        const Enc8 a4 = encode8_slow(x[0].x, x[0].y, x[1].x, x[1].y, x[2].x, x[2].y, x[3].x,
                                     x[3].y, t4.x);
        r.q6 = a6.q; r.e6 = a6.err;
        r.q4 = a4.q; r.e4 = a4.err;
    }
    return r;
}

__device__ __forceinline__ void load_x(const uint4& w, float2* x) {
    const uint32_t u[4] = {w.x, w.y, w.z, w.w};
    const float2 nz = make_float2(-0.0f, -0.0f);              // x + (-0) = x exactly
#pragma unroll
    for (int j = 0; j < 4; ++j) x[j] = bf16x2_add_f32x2(u[j], nz);
}

// 1D: 32 consecutive 16-element blocks of the dense [M][N] matrix per warp and
// step (block b = elements 16 b .. 16 b + 15, a row's blocks followed by the
// next row's since N % 16 == 0), one block per lane (encode_block16: the
// block-level work once, no shuffles): 1 KB contiguous per warp for any N.
__device__ void encode_rows(const MatArgs& a, const MatShared& sh, const EncodeConsts& c,
                            uint64_t release) {
    const int lane = threadIdx.x & 31;
    const long long wg = (long long)blockIdx.x * kMqWarps + (threadIdx.x >> 5);
    const long long nw = (long long)gridDim.x * kMqWarps;
    const long long nblocks = (long long)a.M * (a.N / 16);
    for (long long b0 = wg * 32; b0 < nblocks; b0 += nw * 32) {
        const long long b = b0 + lane;
        const bool valid = b < nblocks;
        uint4 w0 = make_uint4(0u, 0u, 0u, 0u), w1 = w0;
        if (valid) {
            w0 = ld_hint(a.X + 2 * b, release);
            w1 = ld_hint(a.X + 2 * b + 1, release);
        }
        float2 x[8];
        load_x(w0, x);
        load_x(w1, x + 4);
        const float ab = fmaxf(max_abs8(x), max_abs8(x + 4));
        const BlockCodes16 bc = encode_block16(x, ab, sh.tab, c, a.one);
        if (valid) {
            *reinterpret_cast<uint2*>(a.codes + 2 * b) = bc.q;
            a.scales[b] = (uint8_t)bc.sb;
        }
    }
}

// 2D: one 16 x 16 tile per warp; lane = (row lane/2, half lane&1).
__device__ void encode_tiles(const MatArgs& a, const MatShared& sh, const EncodeConsts& c,
                             uint64_t release) {
    const int lane = threadIdx.x & 31;
    const int wg = blockIdx.x * kMqWarps + (threadIdx.x >> 5);
    const int nw = gridDim.x * kMqWarps;
    const int tcols = a.N / 16;
    const int ntiles = (a.M / 16) * tcols;
    const int r = lane >> 1, half = lane & 1;
    for (int u = wg; u < ntiles; u += nw) {
        const int tr = u / tcols;
        const int tc = u - tr * tcols;
        const size_t e0 = (size_t)(tr * 16 + r) * a.N + tc * 16 + half * 8;
        float2 x[4];
        load_x(ld_hint(a.X + e0 / 8, release), x);
        float ab = max_abs8(x);
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) ab = fmaxf(ab, __shfl_xor_sync(0xFFFFFFFFu, ab, o));
        const LaneEnc q = encode_lane(x, ab, sh, c, a.one);
        // row segment = (elements 0..7) + (elements 8..15); tile = rows in order
        const float s6 = __fadd_rn(q.e6, __shfl_xor_sync(0xFFFFFFFFu, q.e6, 1));
        const float s4 = __fadd_rn(q.e4, __shfl_xor_sync(0xFFFFFFFFu, q.e4, 1));
        float E6 = __shfl_sync(0xFFFFFFFFu, s6, 0), E4 = __shfl_sync(0xFFFFFFFFu, s4, 0);
#pragma unroll
        for (int rr = 1; rr < 16; ++rr) {
            E6 = __fadd_rn(E6, __shfl_sync(0xFFFFFFFFu, s6, 2 * rr));
            E4 = __fadd_rn(E4, __shfl_sync(0xFFFFFFFFu, s4, 2 * rr));
        }
        const bool keep4 = E4 < E6;
        uint32_t w = keep4 ? q.q4 : q.q6;
        if (!((keep4 ? q.D4 : q.D6) > 0.0f)) w = 0u;
        a.codes[e0 / 8] = w;
        if (lane == 0) a.scales[u] = (uint8_t)(keep4 ? q.sb4 : q.sb6);
    }
}

__global__ void __launch_bounds__(kMqThreads, 1) matrix_quant_kernel(MatArgs a) {
    __shared__ MatShared sh;
    const uint64_t keep = policy_keep(), release = policy_release();
    phase_amax(a, sh, keep);
    if (!grid_barrier(a.ctl)) return;
    float m = 0.0f;
    for (int i = threadIdx.x; i < gridDim.x; i += blockDim.x) m = fmaxf(m, __ldcg(a.part + i));
    const float A = cta_max(m, sh.red);
    const float s = A > 0.0f ? __fdiv_rn(A, kTensorScaleDiv) : 1.0f;
    if (blockIdx.x == 0 && threadIdx.x == 0) *a.tensor_scale = s;
    for (int c = threadIdx.x; c < 256; c += blockDim.x) {
        const float D = __fmul_rn(e4m3_to_f32((uint32_t)c), s);
        sh.tab[c] = make_float2(D, D > 0.0f ? __frcp_rn(D) : 0.0f);
    }
    __syncthreads();
    const EncodeConsts c = encode_consts(s);
    if (a.mode == 1)
        encode_rows(a, sh, c, release);
    else
        encode_tiles(a, sh, c, release);
}

int g_mq_grid[64];      // cooperative grid size per device ordinal (0 = not yet known)

}  // namespace

size_t matrix_workspace_bytes() { return 256 + align256((size_t)kMaxGrid * 4); }

nvfp4kv_status launch_quantize_matrix(const void* X, int M, int N, int mode, void* codes,
                                      void* scales, float* tensor_scale, void* ws,
                                      cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4KV_ERR_CUDA;
    if (g_mq_grid[dev] == 0) {
        int sms = 0, per_sm = 0;
        if (cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
            return NVFP4KV_ERR_CUDA;
        if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, matrix_quant_kernel,
                                                          kMqThreads, 0) != cudaSuccess ||
            per_sm < 1)
            return NVFP4KV_ERR_CUDA;
        g_mq_grid[dev] = min(sms * per_sm, kMaxGrid);
    }
    MatArgs a;
    a.X = static_cast<const uint4*>(X);
    a.M = M;
    a.N = N;
    a.mode = mode;
    a.codes = static_cast<uint32_t*>(codes);
    a.scales = static_cast<uint8_t*>(scales);
    a.tensor_scale = tensor_scale;
    a.ctl = static_cast<Control*>(ws);
    a.part = reinterpret_cast<float*>(static_cast<char*>(ws) + 256);
    a.one = 1.0f;
    void* args[] = {&a};
    cudaError_t e = cudaLaunchCooperativeKernel((const void*)matrix_quant_kernel,
                                                dim3(g_mq_grid[dev]), dim3(kMqThreads), args, 0,
                                                stream);
    return e == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

}  // namespace nvfp4kv
