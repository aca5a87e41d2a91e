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
// moves 2 bytes in and 2 bytes out per element and is bound by HBM: a thread
// takes 8 channels of one token in every head, reads their four table entries
// once, and keeps 12 heads' 16-byte loads in flight.
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

constexpr int kRopeThreads = 256;
constexpr int kRopeBatch = 12;            // heads whose 16-byte loads are in flight together

// Table entry of head pair P for a token at frame f, row r, column c.
__device__ __forceinline__ int rope_entry(const RopeDev& g, int f, int r, int c, int P) {
    if (P < kRopeRowPair0) return f * kRopeFramePairs + P;
    if (P < kRopeColPair0) return g.frames * kRopeFramePairs + r * kRopeAxisPairs + P - kRopeRowPair0;
    return g.frames * kRopeFramePairs + g.rows * kRopeAxisPairs + c * kRopeAxisPairs + P -
           kRopeColPair0;
}

// Thread = (token t, channel group q): the 8 channels 8 q .. 8 q + 7 (head
// pairs 4 q .. 4 q + 3) of every head of token t.  Their four table entries
// depend on the token and the pairs only, so they are read once (through L1)
// and kept in registers for all H heads; a warp covers two tokens, each head's
// 256 bytes of a token contiguous.
__global__ void __launch_bounds__(kRopeThreads) rope_kernel(const uint4* X, uint4* Y, int T,
                                                            int H, RopeDev g) {
    const int q = threadIdx.x & 15;
    for (int t = (blockIdx.x * blockDim.x + threadIdx.x) >> 4; t < T;
         t += (gridDim.x * blockDim.x) >> 4) {
        const uint4* src = X + (size_t)t * H * 16 + q;
        uint4* dst = Y + (size_t)t * H * 16 + q;
        uint4 w[kRopeBatch];
        // the first heads' loads go out before the table reads they do not need
#pragma unroll
        for (int k = 0; k < kRopeBatch; ++k)
            w[k] = k < H ? __ldcs(src + k * 16) : make_uint4(0u, 0u, 0u, 0u);
        const uint32_t f = rope_div((uint32_t)t, g.m_rc);
        const uint32_t rem = (uint32_t)t - f * (uint32_t)g.rc;
        const uint32_t r = rope_div(rem, g.m_c);
        const uint32_t c = rem - r * (uint32_t)g.cols;
        float2 cs[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) cs[j] = __ldg(g.tab + rope_entry(g, f, r, c, 4 * q + j));
        for (int h0 = 0; h0 < H; h0 += kRopeBatch) {
            if (h0 > 0) {
#pragma unroll
                for (int k = 0; k < kRopeBatch; ++k)
                    w[k] = h0 + k < H ? __ldcs(src + (h0 + k) * 16) : make_uint4(0u, 0u, 0u, 0u);
            }
#pragma unroll
            for (int k = 0; k < kRopeBatch; ++k) {
                if (h0 + k < H) {
                    const uint4 v = make_uint4(rope_pair(w[k].x, cs[0], g.one),
                                               rope_pair(w[k].y, cs[1], g.one),
                                               rope_pair(w[k].z, cs[2], g.one),
                                               rope_pair(w[k].w, cs[3], g.one));
                    __stcs(dst + (h0 + k) * 16, v);
                }
            }
        }
    }
}

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
    const int sms = sm_count_cached();
    if (sms <= 0) return NVFP4KV_ERR_CUDA;
    const long long threads = 16LL * T;
    const long long want = (threads + kRopeThreads - 1) / kRopeThreads;
    const int blocks = (int)(want < 4LL * sms ? want : 4LL * sms);
    rope_kernel<<<blocks, kRopeThreads, 0, stream>>>(static_cast<const uint4*>(X),
                                                     static_cast<uint4*>(Y), T, H, rope_dev(r));
    return cudaGetLastError() == cudaSuccess ? NVFP4KV_OK : NVFP4KV_ERR_CUDA;
}

}  // namespace nvfp4kv
