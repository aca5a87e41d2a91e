// rope.cu -- 3D rotary position embedding of a chunk's queries or keys, with
// the multi-shot frame offset.
//
// The txtmix page "LongLive 2.0：给长视频生成补上 NVFP4 并行基础设施" names a
// fused RoPE kernel on the NVFP4 inference path (section NVFP4：一条从训练贯穿
// 到 KV cache 的量化线) and the option multi_shot_rope_offset, a RoPE position
// offset that keeps the positions of different shots apart (section 多 shot
// 一致性); it gives no rotary form.  The form built here is a reading:
//   - a chunk's tokens form frames of rows x cols latent tokens, frame-major,
//     then row, then column;
//   - a head's 128 channels split into a frame part (channels 0..43), a row
//     part (44..85) and a column part (86..127); in a part of width w the
//     channel pair (2i, 2i+1) turns by p * 10000^(-2i/w), p the token's
//     coordinate on that part's axis;
//   - the frame coordinate is frame_pos0 + the frame within the chunk, and a
//     multi-shot stream starts chunk n of shot s at n * F_c + s * offset;
//   - the frequency, the angle, cos and sin are evaluated in double precision
//     and rounded once to fp32 (the table); the rotation is fp32 with one
//     rounding per product and sum, and the results are rounded to bf16.
//
// Two kernels: the table of a chunk (one thread per entry), and the rotation
// of a bf16 [T][H][128] tensor (the queries; the chunk quantizer rotates K
// itself inside its statistics and encoding passes, quant.cu).  The rotation
// moves 2 bytes in and 2 bytes out per element and is bound by HBM: two CTAs
// per SM stage the table in shared memory (rope.cuh's padded rows), and each
// thread keeps four 16-byte loads in flight.
#include "common.cuh"
#include "kernels.h"
#include "rope.cuh"

namespace nvfp4kv {
namespace {

__global__ void rope_table_kernel(long long frame_pos0, int frames, int rows, int cols,
                                  float2* tab) {
    const int nf = frames * kRopeFramePairs;
    const int nr = rows * kRopeAxisPairs;
    const int n = nf + nr + cols * kRopeAxisPairs;
    for (int e = blockIdx.x * blockDim.x + threadIdx.x; e < n; e += gridDim.x * blockDim.x) {
        long long p;
        int i, w;
        if (e < nf) {
            p = frame_pos0 + e / kRopeFramePairs;
            i = e % kRopeFramePairs;
            w = 2 * kRopeFramePairs;
        } else {
            const int k = e < nf + nr ? e - nf : e - nf - nr;
            p = k / kRopeAxisPairs;
            i = k % kRopeAxisPairs;
            w = 2 * kRopeAxisPairs;
        }
        const double omega = pow(10000.0, (double)(-2 * i) / (double)w);
        const double phi = (double)p * omega;
        tab[e] = make_float2((float)cos(phi), (float)sin(phi));
    }
}

constexpr int kRopeThreads = 512;
constexpr int kRopeUnroll = 4;            // 16-byte loads in flight per thread

// Units of 16 bytes: unit u of X is token (u / 16) / H, channels 8 q .. 8 q + 7
// with q = u % 16 (head pairs 4 q .. 4 q + 3).  The grid stride is a multiple
// of 16, so a thread keeps one q and one pair group.
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(const uint4* X, uint4* Y, int T,
                                                            int H, uint64_t m_h, RopeDev g) {
    extern __shared__ float2 rope_sm[];
    rope_stage(g, rope_sm);
    __syncthreads();
    const uint32_t n16 = (uint32_t)T * (uint32_t)H * 16u;
    const uint32_t stride = gridDim.x * blockDim.x;
    const uint32_t first = blockIdx.x * blockDim.x + threadIdx.x;
    const RopeGroup grp = rope_group(4 * (int)(first & 15u));
    for (uint32_t u0 = first; u0 < n16; u0 += kRopeUnroll * stride) {
        uint4 w[kRopeUnroll];
#pragma unroll
        for (int k = 0; k < kRopeUnroll; ++k) {
            const uint32_t u = u0 + k * stride;
            w[k] = u < n16 ? __ldcs(X + u) : make_uint4(0u, 0u, 0u, 0u);
        }
#pragma unroll
        for (int k = 0; k < kRopeUnroll; ++k) {
            const uint32_t u = u0 + k * stride;
            if (u < n16) {
                uint32_t v[4] = {w[k].x, w[k].y, w[k].z, w[k].w};
                rope_group4(grp, rope_rows(g, rope_div(u >> 4, m_h)), rope_sm, g.one, v);
                __stcs(Y + u, make_uint4(v[0], v[1], v[2], v[3]));
            }
        }
    }
}

bool g_rope_smem_set[64];   // the dynamic shared memory limit raised, per device

}  // namespace

size_t rope_table_entries(int frames, int rows, int cols) {
    return (size_t)frames * kRopeFramePairs + ((size_t)rows + cols) * kRopeAxisPairs;
}

size_t rope_staged_bytes(int frames, int rows, int cols) {
    return (size_t)rope_staged_slots(frames, rows, cols) * sizeof(float2);
}

RopeDev rope_dev(const RopeGeom& r) {
    RopeDev g;
    g.tab = static_cast<const float2*>(r.table);
    g.frames = r.frames;
    g.rows = r.rows;
    g.cols = r.cols;
    g.rc = r.rows * r.cols;
    g.entries = (int)rope_table_entries(r.frames, r.rows, r.cols);
    g.rowslot = r.frames * kRopeFrameRow;
    g.colslot = g.rowslot + r.rows * kRopeRowRow;
    g.m_rc = rope_reciprocal((uint32_t)g.rc);
    g.m_c = rope_reciprocal((uint32_t)r.cols);
    g.one = 1.0f;
    return g;
}

nvfp4kv_status launch_rope_table(long long frame_pos0, int frames, int rows, int cols,
                                 void* table, cudaStream_t stream) {
    const int n = (int)rope_table_entries(frames, rows, cols);
    const int blocks = (n + 255) / 256;
    rope_table_kernel<<<blocks, 256, 0, stream>>>(frame_pos0, frames, rows, cols,
                                                  static_cast<float2*>(table));
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

nvfp4kv_status launch_rope(const void* X, void* Y, int T, int H, const RopeGeom& r,
                           cudaStream_t stream) {
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return NVFP4KV_ERR_CUDA;
    if (!g_rope_smem_set[dev]) {
        if (cudaFuncSetAttribute(rope_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)kRopeMaxStagedBytes) != cudaSuccess)
            return NVFP4KV_ERR_CUDA;
        g_rope_smem_set[dev] = true;
    }
    const int sms = sm_count_cached();
    if (sms <= 0) return NVFP4KV_ERR_CUDA;
    const long long n16 = (long long)T * H * 16;
    const long long per_pass = (long long)kRopeThreads * kRopeUnroll;
    const long long want = (n16 + per_pass - 1) / per_pass;
    const int blocks = (int)(want < 2LL * sms ? want : 2LL * sms);
    rope_kernel<<<blocks, kRopeThreads, rope_staged_bytes(r.frames, r.rows, r.cols), stream>>>(
        static_cast<const uint4*>(X), static_cast<uint4*>(Y), T, H,
        rope_reciprocal((uint32_t)H), rope_dev(r));
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

}  // namespace nvfp4kv
