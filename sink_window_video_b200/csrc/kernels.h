// kernels.h -- host-side entry points of the CUDA kernels (internal to the
// library; the public C ABI is include/nvfp4kv.h).
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>

#include "nvfp4kv.h"

namespace nvfp4kv {

constexpr int kMaxGrid = 4096;       // room for per-CTA partials in the workspace
constexpr int kHeadDimSupported = 128;   // head dimension d the kernels support

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// Attention work split (see attention_plan_tiles): the query blocks that do
// not fill a whole wave of CTAs are split into up to kMaxSplit key ranges,
// whose partial results (per row: 128 fp32 outputs, the running max and the
// row sum) go to the workspace and are merged by a second kernel.
constexpr int kMaxTailPairs = 160;   // 256-row units: more than one wave never remains
constexpr int kMaxSplit = 8;
constexpr int kPartialFloats = 132;  // per row: O[128], m, l, 2 pad (16-byte rows)

// Workspace layout for chunks of T tokens and H heads (d = 128):
//   [0, 256)  Control (status word, grid barrier)
//   psum      float    [nseg][H*d]  per-segment column sums of K
//   pmin/pmax bf16     [nseg][H*d]  per-segment column min / max of K
//   kpart     float    [kMaxGrid]   per-CTA max |K - mean|
//   vpart     float    [kMaxGrid]   per-CTA max |V|
//   (the quantizer uses the workspace up to here: quant_total)
//   apart     float    [tail rows * kMaxSplit][132]  attention partials, room
//             for apart_rows tail rows (a multiple of 256, at least T rounded
//             up to 256 per head, at most 160 x 256)
struct WsLayout {
    size_t psum, pmin, pmax, kpart, vpart, quant_total, apart, apart_rows, total;
};

inline WsLayout ws_layout(int T, int H) {
    size_t HD = (size_t)H * 128;
    size_t nseg = ((size_t)T + 63) / 64;
    WsLayout L;
    size_t off = 256;
    L.psum = off;  off += align256(nseg * HD * 4);
    L.pmin = off;  off += align256(nseg * HD * 2);
    L.pmax = off;  off += align256(nseg * HD * 2);
    L.kpart = off; off += align256(kMaxGrid * 4);
    L.vpart = off; off += align256(kMaxGrid * 4);
    L.quant_total = off;
    const size_t pairs = (size_t)H * (((size_t)T + 255) / 256);
    L.apart_rows = 256 * (pairs < (size_t)kMaxTailPairs ? pairs : (size_t)kMaxTailPairs);
    L.apart = off; off += align256(L.apart_rows * kMaxSplit * kPartialFloats * 4);
    L.total = off;
    return L;
}

// How one attention call is laid out on the GPU: query blocks of block_rows
// rows of one head, n_full of them whole, then n_tail blocks each split into
// n_split key ranges (n_split = 1: no split, no second kernel).  Block b
// covers head b / blocks_per_head, rows (b % blocks_per_head) * block_rows...
struct AttnPlan {
    int block_rows, blocks_per_head, n_blocks, n_full, n_tail, n_split;
};
// The exact attention kernel's plan (attention_ws.cu).
AttnPlan attention_plan(int n_chunks, int T_c, int H, int T_q, size_t tail_capacity_rows);
// The plan for a kernel of `ntiles` key tiles per query block of block_rows rows.
AttnPlan attention_plan_tiles(int ntiles, int H, int T_q, int block_rows,
                              size_t tail_capacity_rows);
// The second kernel of a split plan: merges the partial rows in `part` into O.
nvfp4kv_status launch_attention_merge(const float* part, const AttnPlan& plan, int T_q, int H,
                                      void* O, int o_f32, cudaStream_t stream);

// The queries as NVFP4 rows for the FP4-operand attention: codes
// [T_q * H][64], block scales [T_q * H][8], the FP32 tensor scale.
struct Fp4qLayout {
    size_t codes, scales, scale, total;
};
inline Fp4qLayout fp4q_layout(int T_q, int H) {
    const size_t rows = (size_t)T_q * H;
    Fp4qLayout L;
    L.codes = 0;
    L.scales = align256(rows * 64);
    L.scale = L.scales + align256(rows * 8);
    L.total = L.scale + 256;
    return L;
}

// The argument checks of nvfp4kv_quantize_chunk, in its order (need_ws: the
// workspace pointer is checked too); the no-allocation entry point runs the
// same checks without a workspace.
nvfp4kv_status check_quantize_chunk_args(const void* K, const void* V, int T_c, int H, int d,
                                         const nvfp4kv_chunk_view* out, const void* ws,
                                         bool need_ws);

struct RopeGeom;
// rope: K is rotated (rope.cu's reading) before it is quantized; null for none.
nvfp4kv_status launch_quantize(const void* K, const void* V, int T, int H,
                               const nvfp4kv_chunk_view& out, void* ws, cudaStream_t stream,
                               const RopeGeom* rope = nullptr);

// Sequence-parallel phases of the chunk quantizer (quant.cu).
nvfp4kv_status launch_sp_stats(const void* K, const void* V, int T_local, int H, float* psum,
                               void* pmin, void* pmax, float* vmax, void* ws,
                               cudaStream_t stream);
nvfp4kv_status launch_sp_finalize(const float* psum, const void* pmin, const void* pmax,
                                  int nseg, int T, int H, const float* vmax, float* k_mean,
                                  float* amax, float* tensor_scales, void* ws,
                                  cudaStream_t stream);
nvfp4kv_status launch_scales_from_amax(const float* amax, float* tensor_scales,
                                       cudaStream_t stream);
nvfp4kv_status launch_sp_encode(const void* K, const void* V, int T_local, int H,
                                const float* k_mean, const float* tensor_scales,
                                const nvfp4kv_chunk_view& out, cudaStream_t stream);

// Weight / activation quantizer (matrix_quant.cu): workspace = control block +
// per-CTA partial maxima.
size_t matrix_workspace_bytes();
nvfp4kv_status launch_quantize_matrix(const void* X, int M, int N, int mode, void* codes,
                                      void* scales, float* tensor_scale, void* ws,
                                      cudaStream_t stream);

// 3D rotary position embedding (rope.cu): a chunk's cos/sin table and the
// frame grid of its tokens (frames * rows * cols >= T).
struct RopeGeom {
    const void* table;
    int frames, rows, cols;
};
size_t rope_table_entries(int frames, int rows, int cols);
// Shared memory of a staged table (rope.cuh's padded rows, the chunk
// quantizer's copy); the entry points accept grids up to kRopeMaxStagedBytes.
constexpr size_t kRopeMaxStagedBytes = 61440;
size_t rope_staged_bytes(int frames, int rows, int cols);
nvfp4kv_status launch_rope_table(long long frame_pos0, int frames, int rows, int cols,
                                 void* table, cudaStream_t stream);
nvfp4kv_status launch_rope(const void* X, void* Y, int T, int H, const RopeGeom& r,
                           cudaStream_t stream);

int sm_count_cached();
nvfp4kv_status launch_dequantize(const nvfp4kv_chunk_view& in, int T, int H, void* K_out,
                                 void* V_out, int out_dtype, cudaStream_t stream);

nvfp4kv_status launch_check_formats(int op, const void* in, void* out, size_t n,
                                    cudaStream_t stream);

nvfp4kv_status launch_attention_ws(const nvfp4kv_chunk_view* chunks, int n_chunks, int T_c,
                                   int H, const void* Q, int T_q, void* O, int o_dtype,
                                   float softmax_scale, void* ws, cudaStream_t stream);

// Sink-window attention with the queries quantized to NVFP4 (into q_fp4,
// laid out by fp4q_layout) and Q K^T on the block-scaled FP4 tensor cores
// (attention_fp4.cu); the matrix quantizer runs on ws first.
AttnPlan attention_fp4_plan(int n_chunks, int T_c, int H, int T_q, size_t tail_capacity_rows);
nvfp4kv_status launch_attention_fp4(const nvfp4kv_chunk_view* chunks, int n_chunks, int T_c,
                                    int H, const void* Q, int T_q, void* O, int o_dtype,
                                    float softmax_scale, void* q_fp4, void* ws,
                                    cudaStream_t stream);

// Sink-window attention: the warp-specialized tcgen05 kernel (and its merge
// kernel for split query blocks).
nvfp4kv_status launch_attention(const nvfp4kv_chunk_view* chunks, int n_chunks, int T_c,
                                int H, const void* Q, int T_q, void* O, int o_dtype,
                                float softmax_scale, void* ws, cudaStream_t stream);

}  // namespace nvfp4kv
