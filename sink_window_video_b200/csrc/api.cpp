// api.cpp -- the library's C ABI (include/nvfp4kv.h): argument checks, chunk
// buffer layout, the KV cache manager, and dispatch to the kernels.
//
// Cache manager ("2605-LongLive2" DeepRead page, Method > 算法层设计,
// Multi-Shot Attention Sink): per layer a pool of S_g + S_s + W chunk slots.
// With n chunks appended, the attended set is
//   A_g = [0, S_g),  A_s = [s_begin, s_begin + S_s) n [0, n),  window = [n - W, n),
// de-duplicated by chunk id.  Appending chunk n first frees every slot whose
// chunk is not in the set for n + 1 chunks, then claims a free slot (the live
// set never exceeds the pool).  A prompt switch moves s_begin (two pointers,
// no device memory); chunks of the old shot sink are freed once they are
// outside the window.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "kernels.h"
#include "nvfp4kv.h"

using namespace nvfp4kv;

struct kvcache {
    kvcache_config cfg;
    int slots;
    size_t chunk_bytes;
    uint8_t* pool;
    void* ws;
    int64_t s_begin;
    bool ws_ready;                     // control words zeroed on a stream
    std::vector<int64_t> n;            // chunks appended, per layer
    std::vector<int64_t> slot_chunk;   // [layer * slots + slot] -> chunk id or -1
};

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned256(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 255u) == 0; }

bool valid_shape(int T, int H, int d) {
    return T > 0 && H > 0 && d > 0 && d % 16 == 0 && T <= (1 << 24) && H <= 4096 &&
           (size_t)T * H * d < ((size_t)1 << 34);
}

struct ChunkLayout {
    size_t k_codes, v_codes, k_scales, v_scales, k_mean, tscale, total;
};

ChunkLayout chunk_layout(int T, int H, int d) {
    const size_t n = (size_t)T * H * d;
    ChunkLayout L;
    size_t off = 0;
    L.k_codes = off;  off += align256(n / 2);
    L.v_codes = off;  off += align256(n / 2);
    L.k_scales = off; off += align256(n / 16);
    L.v_scales = off; off += align256(n / 16);
    L.k_mean = off;   off += align256((size_t)H * d * 4);
    L.tscale = off;   off += 256;
    L.total = off;
    return L;
}

nvfp4kv_chunk_view carve(uint8_t* base, const ChunkLayout& L) {
    nvfp4kv_chunk_view v;
    v.k_codes = base + L.k_codes;
    v.v_codes = base + L.v_codes;
    v.k_scales = base + L.k_scales;
    v.v_scales = base + L.v_scales;
    v.k_mean = reinterpret_cast<float*>(base + L.k_mean);
    v.tensor_scales = reinterpret_cast<float*>(base + L.tscale);
    return v;
}

bool view_ok(const nvfp4kv_chunk_view& v) {
    return v.k_codes && v.k_scales && v.v_codes && v.v_scales && v.k_mean && v.tensor_scales &&
           aligned16(v.k_codes) && aligned16(v.v_codes) && aligned16(v.k_mean) &&
           aligned16(v.k_scales) && aligned16(v.v_scales) &&
           (reinterpret_cast<uintptr_t>(v.tensor_scales) & 7u) == 0;
}

// Attended chunk ids after n appends: sorted, unique.
void keyset_ids(const kvcache* c, int64_t n, std::vector<int64_t>& ids) {
    ids.clear();
    const kvcache_config& k = c->cfg;
    for (int64_t id = 0; id < std::min<int64_t>(k.S_g, n); ++id) ids.push_back(id);
    for (int64_t id = c->s_begin; id < c->s_begin + k.S_s; ++id)
        if (id >= 0 && id < n) ids.push_back(id);
    for (int64_t id = std::max<int64_t>(0, n - k.W); id < n; ++id) ids.push_back(id);
    std::sort(ids.begin(), ids.end());
    ids.erase(std::unique(ids.begin(), ids.end()), ids.end());
}

int find_slot(const kvcache* c, int layer, int64_t chunk) {
    const int64_t* sc = &c->slot_chunk[(size_t)layer * c->slots];
    for (int s = 0; s < c->slots; ++s)
        if (sc[s] == chunk) return s;
    return -1;
}

nvfp4kv_chunk_view slot_view(const kvcache* c, int layer, int slot) {
    const ChunkLayout L = chunk_layout(c->cfg.T_c, c->cfg.H, c->cfg.d);
    return carve(c->pool + ((size_t)layer * c->slots + slot) * c->chunk_bytes, L);
}

bool have_sm100() {
    static int state = -1;
    if (state < 0) {
        int dev = 0, major = 0;
        state = (cudaGetDevice(&dev) == cudaSuccess &&
                 cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) ==
                     cudaSuccess &&
                 major == 10)
                    ? 1
                    : 0;
    }
    return state == 1;
}

// A rotation's grid: every size at least 1, rows*cols < 2^16 and at most
// 2^20 frames (the table's index and the token division stay in 32 bits).
bool rope_grid_ok(int frames, int rows, int cols) {
    return frames >= 1 && rows >= 1 && cols >= 1 && frames <= (1 << 20) &&
           (long long)rows * cols <= 65535;
}

// The rotation of T tokens: a valid view whose table covers them and fits the
// consumers' shared memory when staged.
nvfp4kv_status check_rope_view(const nvfp4kv_rope_view* r, int T) {
    if (!r || !r->table || !rope_grid_ok(r->frames, r->rows, r->cols) || T > 65535 ||
        (long long)r->frames * r->rows * r->cols < T ||
        nvfp4kv::rope_staged_bytes(r->frames, r->rows, r->cols) > nvfp4kv::kRopeMaxStagedBytes)
        return NVFP4KV_ERR_INVALID_ARG;
    if (!aligned16(r->table)) return NVFP4KV_ERR_ALIGNMENT;
    return NVFP4KV_OK;
}

nvfp4kv::RopeGeom rope_geom(const nvfp4kv_rope_view& r) {
    nvfp4kv::RopeGeom g;
    g.table = r.table;
    g.frames = r.frames;
    g.rows = r.rows;
    g.cols = r.cols;
    return g;
}

}  // namespace

namespace nvfp4kv {
nvfp4kv_status check_quantize_chunk_args(const void* K, const void* V, int T_c, int H, int d,
                                         const nvfp4kv_chunk_view* out, const void* ws,
                                         bool need_ws) {
    if (!K || !V || !out || (need_ws && !ws) || !valid_shape(T_c, H, d) || !view_ok(*out))
        return NVFP4KV_ERR_INVALID_ARG;
    if (d != kHeadDimSupported) return NVFP4KV_ERR_UNSUPPORTED;
    if (!aligned16(K) || !aligned16(V) || (need_ws && !aligned256(ws)))
        return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return NVFP4KV_OK;
}

nvfp4kv_status launch_attention(const nvfp4kv_chunk_view* chunks, int n_chunks, int T_c, int H,
                                const void* Q, int T_q, void* O, int o_dtype, float softmax_scale,
                                void* ws, cudaStream_t stream) {
    return launch_attention_ws(chunks, n_chunks, T_c, H, Q, T_q, O, o_dtype, softmax_scale, ws,
                               stream);
}
}  // namespace nvfp4kv

extern "C" {

const char* nvfp4kv_version(void) { return "nvfp4kv 0.1 (sm_100a)"; }

size_t nvfp4kv_chunk_bytes(int T_c, int H, int d) {
    if (!valid_shape(T_c, H, d)) return 0;
    return chunk_layout(T_c, H, d).total;
}

nvfp4kv_status nvfp4kv_chunk_view_init(void* base, int T_c, int H, int d,
                                       nvfp4kv_chunk_view* out) {
    if (!base || !out || !valid_shape(T_c, H, d)) return NVFP4KV_ERR_INVALID_ARG;
    if (!aligned256(base)) return NVFP4KV_ERR_ALIGNMENT;
    *out = carve(static_cast<uint8_t*>(base), chunk_layout(T_c, H, d));
    return NVFP4KV_OK;
}

int nvfp4kv_attention_launches(int n_chunks, int T_c, int H, int d, int T_q) {
    if (!valid_shape(T_c, H, d) || n_chunks < 1 || n_chunks > NVFP4KV_MAX_KEY_CHUNKS ||
        T_q <= 0)
        return 0;
    const AttnPlan p = attention_plan(n_chunks, T_c, H, T_q, ws_layout(T_c, H).apart_rows);
    return p.n_tail > 0 ? 2 : 1;
}

size_t nvfp4kv_workspace_bytes(int T_c, int H, int d) {
    if (!valid_shape(T_c, H, d)) return 0;
    return ws_layout(T_c, H).total;
}

nvfp4kv_status nvfp4kv_workspace_init(void* ws, size_t ws_bytes, nvfp4kv_stream_t stream) {
    if (!ws || ws_bytes < 256) return NVFP4KV_ERR_INVALID_ARG;
    if (!aligned256(ws)) return NVFP4KV_ERR_ALIGNMENT;
    return cudaMemsetAsync(ws, 0, 256, (cudaStream_t)stream) == cudaSuccess ? NVFP4KV_OK
                                                                             : NVFP4KV_ERR_CUDA;
}

nvfp4kv_status nvfp4kv_workspace_status(void* ws, nvfp4kv_stream_t stream) {
    if (!ws) return NVFP4KV_ERR_INVALID_ARG;
    unsigned st = 0;
    cudaStream_t s = (cudaStream_t)stream;
    if (cudaMemcpyAsync(&st, ws, sizeof(unsigned), cudaMemcpyDeviceToHost, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return NVFP4KV_ERR_CUDA;
    if (st == 0) return NVFP4KV_OK;
    if (cudaMemsetAsync(ws, 0, sizeof(unsigned), s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
        return NVFP4KV_ERR_CUDA;
    // a wait that gave up outranks an input the attention could not represent
    return (st & 1u) ? NVFP4KV_ERR_DEVICE_TIMEOUT : NVFP4KV_ERR_UNSUPPORTED;
}

nvfp4kv_status nvfp4kv_quantize_chunk(const void* K, const void* V, int T_c, int H, int d,
                                      const nvfp4kv_chunk_view* out, void* ws,
                                      nvfp4kv_stream_t stream) {
    const nvfp4kv_status st = check_quantize_chunk_args(K, V, T_c, H, d, out, ws, true);
    if (st != NVFP4KV_OK) return st;
    return launch_quantize(K, V, T_c, H, *out, ws, (cudaStream_t)stream);
}

long long nvfp4kv_rope_frame_position(long long chunk, int frames_per_chunk, long long shot,
                                      long long offset) {
    if (chunk < 0 || frames_per_chunk < 1 || shot < 0 || offset < 0) return -1;
    return chunk * frames_per_chunk + shot * offset;
}

size_t nvfp4kv_rope_table_bytes(int frames, int rows, int cols) {
    if (!rope_grid_ok(frames, rows, cols)) return 0;
    return 8 * rope_table_entries(frames, rows, cols);
}

nvfp4kv_status nvfp4kv_rope_table(long long frame_pos0, int frames, int rows, int cols,
                                  void* table, nvfp4kv_stream_t stream) {
    if (!table || !rope_grid_ok(frames, rows, cols) || frame_pos0 < 0 ||
        frame_pos0 > (1LL << 40))
        return NVFP4KV_ERR_INVALID_ARG;
    if (!aligned16(table)) return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return launch_rope_table(frame_pos0, frames, rows, cols, table, (cudaStream_t)stream);
}

nvfp4kv_status nvfp4kv_rope(const void* X, void* Y, int T, int H, int d,
                            const nvfp4kv_rope_view* rope, nvfp4kv_stream_t stream) {
    if (!X || !Y || !valid_shape(T, H, d) || (long long)T * H * H >= (1LL << 32))
        return NVFP4KV_ERR_INVALID_ARG;
    {
        // Y == X rotates in place (each 16 bytes read and written by one
        // thread); any other overlap would let a write land before a read
        const uintptr_t x0 = reinterpret_cast<uintptr_t>(X), y0 = reinterpret_cast<uintptr_t>(Y);
        const uintptr_t n = (uintptr_t)T * H * d * 2;
        if (x0 != y0 && x0 < y0 + n && y0 < x0 + n) return NVFP4KV_ERR_INVALID_ARG;
    }
    const nvfp4kv_status st = check_rope_view(rope, T);
    if (st != NVFP4KV_OK) return st;
    if (d != kHeadDimSupported) return NVFP4KV_ERR_UNSUPPORTED;
    if (!aligned16(X) || !aligned16(Y)) return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return launch_rope(X, Y, T, H, rope_geom(*rope), (cudaStream_t)stream);
}

nvfp4kv_status nvfp4kv_quantize_chunk_rope(const void* K, const void* V, int T_c, int H,
                                           int d, const nvfp4kv_rope_view* rope,
                                           const nvfp4kv_chunk_view* out, void* ws,
                                           nvfp4kv_stream_t stream) {
    nvfp4kv_status st = check_rope_view(rope, T_c);
    if (st != NVFP4KV_OK) return st;
    st = check_quantize_chunk_args(K, V, T_c, H, d, out, ws, true);
    if (st != NVFP4KV_OK) return st;
    const RopeGeom g = rope_geom(*rope);
    return launch_quantize(K, V, T_c, H, *out, ws, (cudaStream_t)stream, &g);
}

nvfp4kv_status nvfp4kv_chunk_stats(const void* K, const void* V, int T_local, int H, int d,
                                   float* psum, void* pmin, void* pmax, float* vmax, void* ws,
                                   nvfp4kv_stream_t stream) {
    if (!K || !V || !psum || !pmin || !pmax || !vmax || !ws || !valid_shape(T_local, H, d))
        return NVFP4KV_ERR_INVALID_ARG;
    if (d != kHeadDimSupported) return NVFP4KV_ERR_UNSUPPORTED;
    if (!aligned16(K) || !aligned16(V) || !aligned16(psum) || !aligned16(pmin) ||
        !aligned16(pmax) || !aligned256(ws) || (reinterpret_cast<uintptr_t>(vmax) & 3u) != 0)
        return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return launch_sp_stats(K, V, T_local, H, psum, pmin, pmax, vmax, ws, (cudaStream_t)stream);
}

nvfp4kv_status nvfp4kv_chunk_finalize(const float* psum, const void* pmin, const void* pmax,
                                      int nseg, int T, int H, int d, const float* vmax,
                                      float* k_mean, float* tensor_scales, void* ws,
                                      nvfp4kv_stream_t stream) {
    if (!psum || !pmin || !pmax || !vmax || !k_mean || !tensor_scales || !ws ||
        !valid_shape(T, H, d) || nseg != (T + 63) / 64)
        return NVFP4KV_ERR_INVALID_ARG;
    if (d != kHeadDimSupported) return NVFP4KV_ERR_UNSUPPORTED;
    if (!aligned256(ws) || (reinterpret_cast<uintptr_t>(k_mean) & 15u) != 0)
        return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return launch_sp_finalize(psum, pmin, pmax, nseg, T, H, vmax, k_mean, nullptr,
                              tensor_scales, ws, (cudaStream_t)stream);
}

nvfp4kv_status nvfp4kv_chunk_amax(const float* psum, const void* pmin, const void* pmax,
                                  int nseg, int T, int H, int d, const float* vmax,
                                  float* k_mean, float* amax, void* ws,
                                  nvfp4kv_stream_t stream) {
    if (!psum || !pmin || !pmax || !vmax || !k_mean || !amax || !ws || !valid_shape(T, H, d) ||
        nseg != (T + 63) / 64)
        return NVFP4KV_ERR_INVALID_ARG;
    if (d != kHeadDimSupported) return NVFP4KV_ERR_UNSUPPORTED;
    if (!aligned256(ws) || (reinterpret_cast<uintptr_t>(k_mean) & 15u) != 0)
        return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return launch_sp_finalize(psum, pmin, pmax, nseg, T, H, vmax, k_mean, amax, nullptr, ws,
                              (cudaStream_t)stream);
}

nvfp4kv_status nvfp4kv_tensor_scales_from_amax(const float* amax, float* tensor_scales,
                                               nvfp4kv_stream_t stream) {
    if (!amax || !tensor_scales) return NVFP4KV_ERR_INVALID_ARG;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return launch_scales_from_amax(amax, tensor_scales, (cudaStream_t)stream);
}

nvfp4kv_status nvfp4kv_chunk_encode(const void* K, const void* V, int T_local, int H, int d,
                                    const float* k_mean, const float* tensor_scales,
                                    const nvfp4kv_chunk_view* out, nvfp4kv_stream_t stream) {
    if (!K || !V || !k_mean || !tensor_scales || !out || !valid_shape(T_local, H, d) ||
        !out->k_codes || !out->k_scales || !out->v_codes || !out->v_scales)
        return NVFP4KV_ERR_INVALID_ARG;
    if (d != kHeadDimSupported) return NVFP4KV_ERR_UNSUPPORTED;
    if (!aligned16(K) || !aligned16(V) || !aligned16(out->k_codes) || !aligned16(out->v_codes) ||
        (reinterpret_cast<uintptr_t>(k_mean) & 15u) != 0)
        return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return launch_sp_encode(K, V, T_local, H, k_mean, tensor_scales, *out, (cudaStream_t)stream);
}

size_t nvfp4kv_matrix_workspace_bytes(void) { return matrix_workspace_bytes(); }

nvfp4kv_status nvfp4kv_quantize_matrix(const void* X, int M, int N, int mode, void* codes,
                                       void* scales, float* tensor_scale, void* ws,
                                       nvfp4kv_stream_t stream) {
    if (!X || !codes || !scales || !tensor_scale || !ws || M <= 0 || N <= 0 ||
        (mode != NVFP4KV_BLOCKS_1D && mode != NVFP4KV_TILES_2D) || M > (1 << 24) ||
        N > (1 << 24) || (long long)M * N > (1ll << 34))
        return NVFP4KV_ERR_INVALID_ARG;
    if (N % 16 != 0 || (mode == NVFP4KV_TILES_2D && M % 16 != 0)) return NVFP4KV_ERR_UNSUPPORTED;
    if (!aligned16(X) || !aligned16(codes) || !aligned256(ws) ||
        (reinterpret_cast<uintptr_t>(tensor_scale) & 3u) != 0)
        return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return launch_quantize_matrix(X, M, N, mode, codes, scales, tensor_scale, ws,
                                  (cudaStream_t)stream);
}

nvfp4kv_status nvfp4kv_dequantize(const nvfp4kv_chunk_view* in, int T_c, int H, int d,
                                  void* K_out, void* V_out, int out_dtype,
                                  nvfp4kv_stream_t stream) {
    if (!in || !valid_shape(T_c, H, d) || !view_ok(*in) ||
        (out_dtype != NVFP4KV_F32 && out_dtype != NVFP4KV_BF16))
        return NVFP4KV_ERR_INVALID_ARG;
    if (d != kHeadDimSupported) return NVFP4KV_ERR_UNSUPPORTED;
    if ((K_out && !aligned16(K_out)) || (V_out && !aligned16(V_out))) return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return launch_dequantize(*in, T_c, H, K_out, V_out, out_dtype, (cudaStream_t)stream);
}

nvfp4kv_status nvfp4kv_attention(const nvfp4kv_chunk_view* chunks, int n_chunks, int T_c, int H,
                                 int d, const void* Q, int T_q, void* O, int o_dtype,
                                 float softmax_scale, void* ws, nvfp4kv_stream_t stream) {
    if (!chunks || !Q || !O || !ws || T_q <= 0 || !valid_shape(T_c, H, d) ||
        !valid_shape(T_q, H, d) || (o_dtype != NVFP4KV_F32 && o_dtype != NVFP4KV_BF16))
        return NVFP4KV_ERR_INVALID_ARG;
    if (n_chunks <= 0) return NVFP4KV_ERR_EMPTY_KEYSET;
    if (n_chunks > NVFP4KV_MAX_KEY_CHUNKS) return NVFP4KV_ERR_CAPACITY;
    for (int i = 0; i < n_chunks; ++i)
        if (!view_ok(chunks[i])) return NVFP4KV_ERR_INVALID_ARG;
    if (d != kHeadDimSupported) return NVFP4KV_ERR_UNSUPPORTED;
    if (!aligned16(Q) || !aligned16(O) || !aligned256(ws)) return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    if (!(softmax_scale > 0.0f)) softmax_scale = 1.0f / std::sqrt((float)d);
    return launch_attention(chunks, n_chunks, T_c, H, Q, T_q, O, o_dtype, softmax_scale, ws,
                            (cudaStream_t)stream);
}

size_t nvfp4kv_fp4q_bytes(int T_q, int H, int d) {
    if (!valid_shape(T_q, H, d) || d != kHeadDimSupported) return 0;
    return fp4q_layout(T_q, H).total;
}

nvfp4kv_status nvfp4kv_attention_fp4q(const nvfp4kv_chunk_view* chunks, int n_chunks, int T_c,
                                      int H, int d, const void* Q, int T_q, void* O,
                                      int o_dtype, float softmax_scale, void* q_fp4, void* ws,
                                      nvfp4kv_stream_t stream) {
    if (!chunks || !Q || !O || !q_fp4 || !ws || T_q <= 0 || !valid_shape(T_c, H, d) ||
        !valid_shape(T_q, H, d) || (o_dtype != NVFP4KV_F32 && o_dtype != NVFP4KV_BF16))
        return NVFP4KV_ERR_INVALID_ARG;
    if (n_chunks <= 0) return NVFP4KV_ERR_EMPTY_KEYSET;
    if (n_chunks > NVFP4KV_MAX_KEY_CHUNKS) return NVFP4KV_ERR_CAPACITY;
    for (int i = 0; i < n_chunks; ++i)
        if (!view_ok(chunks[i])) return NVFP4KV_ERR_INVALID_ARG;
    if (d != kHeadDimSupported) return NVFP4KV_ERR_UNSUPPORTED;
    if (!aligned16(Q) || !aligned16(O) || !aligned256(q_fp4) || !aligned256(ws))
        return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    if (!(softmax_scale > 0.0f)) softmax_scale = 1.0f / std::sqrt((float)d);
    return launch_attention_fp4(chunks, n_chunks, T_c, H, Q, T_q, O, o_dtype, softmax_scale,
                                q_fp4, ws, (cudaStream_t)stream);
}

int nvfp4kv_attention_fp4q_launches(int n_chunks, int T_c, int H, int d, int T_q) {
    if (n_chunks <= 0 || n_chunks > NVFP4KV_MAX_KEY_CHUNKS || !valid_shape(T_c, H, d) ||
        d != kHeadDimSupported || T_q <= 0)
        return 0;
    const AttnPlan p = attention_fp4_plan(n_chunks, T_c, H, T_q, ws_layout(T_c, H).apart_rows);
    return 2 + (p.n_tail > 0 ? 1 : 0);
}

nvfp4kv_status nvfp4kv_check_formats(int op, const void* in, void* out, size_t n,
                                     nvfp4kv_stream_t stream) {
    if (!in || !out || op < 0 || op > 5) return NVFP4KV_ERR_INVALID_ARG;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    return launch_check_formats(op, in, out, n, (cudaStream_t)stream);
}

// ---------------------------------------------------------------- cache

size_t kvcache_pool_bytes(const kvcache_config* cfg) {
    if (!cfg || cfg->layers <= 0 || cfg->S_g < 0 || cfg->S_s < 0 || cfg->W < 0) return 0;
    const size_t cb = nvfp4kv_chunk_bytes(cfg->T_c, cfg->H, cfg->d);
    if (!cb) return 0;
    const int slots = std::max(1, cfg->S_g + cfg->S_s + cfg->W);
    return cb * (size_t)slots * (size_t)cfg->layers;
}

nvfp4kv_status kvcache_create(const kvcache_config* cfg, void* pool, void* ws, kvcache** out) {
    if (!out) return NVFP4KV_ERR_INVALID_ARG;
    *out = nullptr;
    if (!cfg || !pool || !ws || kvcache_pool_bytes(cfg) == 0) return NVFP4KV_ERR_INVALID_ARG;
    if (cfg->S_g + cfg->S_s + cfg->W > NVFP4KV_MAX_KEY_CHUNKS) return NVFP4KV_ERR_CAPACITY;
    if (!aligned256(pool) || !aligned256(ws)) return NVFP4KV_ERR_ALIGNMENT;
    kvcache* c = new (std::nothrow) kvcache();
    if (!c) return NVFP4KV_ERR_CAPACITY;
    c->cfg = *cfg;
    c->slots = std::max(1, cfg->S_g + cfg->S_s + cfg->W);
    c->chunk_bytes = nvfp4kv_chunk_bytes(cfg->T_c, cfg->H, cfg->d);
    c->pool = static_cast<uint8_t*>(pool);
    c->ws = ws;
    c->s_begin = 0;
    c->n.assign(cfg->layers, 0);
    c->slot_chunk.assign((size_t)cfg->layers * c->slots, -1);
    c->ws_ready = false;
    *out = c;
    return NVFP4KV_OK;
}

void kvcache_destroy(kvcache* cache) { delete cache; }

nvfp4kv_status kvcache_rebind_shot_sink(kvcache* cache, int64_t first_chunk_of_shot) {
    if (!cache || first_chunk_of_shot < 0) return NVFP4KV_ERR_INVALID_ARG;
    // every chunk of the new shot sink that a layer has appended already must
    // still be stored in that layer (it cannot be brought back)
    for (int layer = 0; layer < cache->cfg.layers; ++layer) {
        const int64_t end = std::min<int64_t>(first_chunk_of_shot + cache->cfg.S_s, cache->n[layer]);
        for (int64_t c = first_chunk_of_shot; c < end; ++c)
            if (find_slot(cache, layer, c) < 0) return NVFP4KV_ERR_INVALID_ARG;
    }
    cache->s_begin = first_chunk_of_shot;
    return NVFP4KV_OK;
}

nvfp4kv_status kvcache_keyset(const kvcache* cache, int layer, int64_t* ids, int* count) {
    if (!cache || !ids || !count) return NVFP4KV_ERR_INVALID_ARG;
    if (layer < 0 || layer >= cache->cfg.layers) return NVFP4KV_ERR_CAPACITY;
    std::vector<int64_t> v;
    keyset_ids(cache, cache->n[layer], v);
    for (size_t i = 0; i < v.size(); ++i) ids[i] = v[i];
    *count = (int)v.size();
    return NVFP4KV_OK;
}

nvfp4kv_status kvcache_num_chunks(const kvcache* cache, int layer, int64_t* n) {
    if (!cache || !n) return NVFP4KV_ERR_INVALID_ARG;
    if (layer < 0 || layer >= cache->cfg.layers) return NVFP4KV_ERR_CAPACITY;
    *n = cache->n[layer];
    return NVFP4KV_OK;
}

nvfp4kv_status kvcache_chunk_view(const kvcache* cache, int layer, int64_t chunk,
                                  nvfp4kv_chunk_view* out) {
    if (!cache || !out) return NVFP4KV_ERR_INVALID_ARG;
    if (layer < 0 || layer >= cache->cfg.layers) return NVFP4KV_ERR_CAPACITY;
    const int s = find_slot(cache, layer, chunk);
    if (s < 0) return NVFP4KV_ERR_INVALID_ARG;
    *out = slot_view(cache, layer, s);
    return NVFP4KV_OK;
}

nvfp4kv_status kvcache_advance(kvcache* cache, int layer, nvfp4kv_chunk_view* out) {
    if (!cache || !out) return NVFP4KV_ERR_INVALID_ARG;
    if (layer < 0 || layer >= cache->cfg.layers) return NVFP4KV_ERR_CAPACITY;
    std::memset(out, 0, sizeof(*out));
    const int64_t n = cache->n[layer];
    std::vector<int64_t> live;
    keyset_ids(cache, n + 1, live);
    int64_t* sc = &cache->slot_chunk[(size_t)layer * cache->slots];
    for (int s = 0; s < cache->slots; ++s)
        if (sc[s] >= 0 && !std::binary_search(live.begin(), live.end(), sc[s])) sc[s] = -1;
    cache->n[layer] = n + 1;
    if (!std::binary_search(live.begin(), live.end(), n)) return NVFP4KV_OK;   // not stored
    for (int s = 0; s < cache->slots; ++s) {
        if (sc[s] < 0) {
            sc[s] = n;
            *out = slot_view(cache, layer, s);
            return NVFP4KV_OK;
        }
    }
    return NVFP4KV_ERR_CAPACITY;    // unreachable: the live set fits the pool
}

namespace {
constexpr uint32_t kStateVersion = 1;
constexpr size_t kStateHeader = 4 + 4 + 7 * 4 + 8;      // tag, version, config, shot sink
}  // namespace

size_t kvcache_state_bytes(const kvcache* cache) {
    if (!cache) return 0;
    return kStateHeader + 8 * (size_t)cache->cfg.layers * (1 + (size_t)cache->slots);
}

nvfp4kv_status kvcache_get_state(const kvcache* cache, void* buf, size_t bytes) {
    if (!cache || !buf || bytes < kvcache_state_bytes(cache)) return NVFP4KV_ERR_INVALID_ARG;
    uint8_t* p = static_cast<uint8_t*>(buf);
    std::memcpy(p, "NVKV", 4);
    std::memcpy(p + 4, &kStateVersion, 4);
    const int32_t cfg[7] = {cache->cfg.layers, cache->cfg.H, cache->cfg.d, cache->cfg.T_c,
                            cache->cfg.S_g,    cache->cfg.S_s, cache->cfg.W};
    std::memcpy(p + 8, cfg, sizeof(cfg));
    std::memcpy(p + 36, &cache->s_begin, 8);
    std::memcpy(p + kStateHeader, cache->n.data(), 8 * cache->n.size());
    std::memcpy(p + kStateHeader + 8 * cache->n.size(), cache->slot_chunk.data(),
                8 * cache->slot_chunk.size());
    return NVFP4KV_OK;
}

nvfp4kv_status kvcache_set_state(kvcache* cache, const void* buf, size_t bytes) {
    if (!cache || !buf || bytes < kvcache_state_bytes(cache)) return NVFP4KV_ERR_INVALID_ARG;
    const uint8_t* p = static_cast<const uint8_t*>(buf);
    uint32_t version = 0;
    std::memcpy(&version, p + 4, 4);
    if (std::memcmp(p, "NVKV", 4) != 0 || version != kStateVersion) return NVFP4KV_ERR_INVALID_ARG;
    int32_t cfg[7];
    std::memcpy(cfg, p + 8, sizeof(cfg));
    const int32_t want[7] = {cache->cfg.layers, cache->cfg.H, cache->cfg.d, cache->cfg.T_c,
                             cache->cfg.S_g,    cache->cfg.S_s, cache->cfg.W};
    if (std::memcmp(cfg, want, sizeof(cfg)) != 0) return NVFP4KV_ERR_INVALID_ARG;
    kvcache next = *cache;
    std::memcpy(&next.s_begin, p + 36, 8);
    std::memcpy(next.n.data(), p + kStateHeader, 8 * next.n.size());
    std::memcpy(next.slot_chunk.data(), p + kStateHeader + 8 * next.n.size(),
                8 * next.slot_chunk.size());
    if (next.s_begin < 0) return NVFP4KV_ERR_INVALID_ARG;
    for (int layer = 0; layer < next.cfg.layers; ++layer) {
        // (a slot may still hold a chunk that left the key set at a shot-sink
        // rebind: the next append frees it)
        const int64_t n = next.n[layer];
        if (n < 0) return NVFP4KV_ERR_INVALID_ARG;
        const int64_t* sc = &next.slot_chunk[(size_t)layer * next.slots];
        std::vector<int64_t> held;
        for (int s = 0; s < next.slots; ++s) {
            if (sc[s] == -1) continue;
            if (sc[s] < 0 || sc[s] >= n) return NVFP4KV_ERR_INVALID_ARG;
            held.push_back(sc[s]);
        }
        std::sort(held.begin(), held.end());
        if (std::adjacent_find(held.begin(), held.end()) != held.end())
            return NVFP4KV_ERR_INVALID_ARG;
    }
    cache->s_begin = next.s_begin;
    cache->n = next.n;
    cache->slot_chunk = next.slot_chunk;
    return NVFP4KV_OK;
}

namespace {
nvfp4kv_status cache_append(kvcache* cache, int layer, const void* K, const void* V,
                            const nvfp4kv_rope_view* rope, nvfp4kv_stream_t stream) {
    if (!cache || !K || !V) return NVFP4KV_ERR_INVALID_ARG;
    if (rope) {
        const nvfp4kv_status r = check_rope_view(rope, cache->cfg.T_c);
        if (r != NVFP4KV_OK) return r;
    }
    if (layer < 0 || layer >= cache->cfg.layers) return NVFP4KV_ERR_CAPACITY;
    if (cache->cfg.d != kHeadDimSupported) return NVFP4KV_ERR_UNSUPPORTED;
    if (!aligned16(K) || !aligned16(V)) return NVFP4KV_ERR_ALIGNMENT;
    if (!have_sm100()) return NVFP4KV_ERR_UNSUPPORTED;
    if (!cache->ws_ready) {
        nvfp4kv_status z = nvfp4kv_workspace_init(cache->ws, 256, stream);
        if (z != NVFP4KV_OK) return z;
        cache->ws_ready = true;
    }
    nvfp4kv_chunk_view v;
    nvfp4kv_status st = kvcache_advance(cache, layer, &v);
    if (st != NVFP4KV_OK || v.k_codes == nullptr) return st;
    if (!rope)
        return launch_quantize(K, V, cache->cfg.T_c, cache->cfg.H, v, cache->ws,
                               (cudaStream_t)stream);
    const RopeGeom g = rope_geom(*rope);
    return launch_quantize(K, V, cache->cfg.T_c, cache->cfg.H, v, cache->ws,
                           (cudaStream_t)stream, &g);
}
}  // namespace

nvfp4kv_status kvcache_append(kvcache* cache, int layer, const void* K, const void* V,
                              nvfp4kv_stream_t stream) {
    return cache_append(cache, layer, K, V, nullptr, stream);
}

nvfp4kv_status kvcache_append_rope(kvcache* cache, int layer, const void* K, const void* V,
                                   const nvfp4kv_rope_view* rope, nvfp4kv_stream_t stream) {
    if (!rope) return NVFP4KV_ERR_INVALID_ARG;
    return cache_append(cache, layer, K, V, rope, stream);
}

nvfp4kv_status sink_window_attention(const kvcache* cache, int layer, const void* Q, int T_q,
                                     void* O, int o_dtype, float softmax_scale,
                                     nvfp4kv_stream_t stream) {
    if (!cache || !Q || !O || T_q <= 0) return NVFP4KV_ERR_INVALID_ARG;
    if (layer < 0 || layer >= cache->cfg.layers) return NVFP4KV_ERR_CAPACITY;
    std::vector<int64_t> ids;
    keyset_ids(cache, cache->n[layer], ids);
    if (ids.empty()) return NVFP4KV_ERR_EMPTY_KEYSET;
    if (ids.size() > NVFP4KV_MAX_KEY_CHUNKS) return NVFP4KV_ERR_CAPACITY;
    nvfp4kv_chunk_view views[NVFP4KV_MAX_KEY_CHUNKS];
    for (size_t i = 0; i < ids.size(); ++i) {
        const int s = find_slot(cache, layer, ids[i]);
        if (s < 0) return NVFP4KV_ERR_INVALID_ARG;    // a stored chunk went missing
        views[i] = slot_view(cache, layer, s);
    }
    return nvfp4kv_attention(views, (int)ids.size(), cache->cfg.T_c, cache->cfg.H, cache->cfg.d,
                             Q, T_q, O, o_dtype, softmax_scale, cache->ws, stream);
}

nvfp4kv_status kvcache_check_status(kvcache* cache, nvfp4kv_stream_t stream) {
    if (!cache) return NVFP4KV_ERR_INVALID_ARG;
    return nvfp4kv_workspace_status(cache->ws, stream);
}

}  // extern "C"
