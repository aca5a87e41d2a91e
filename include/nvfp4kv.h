/*
 * nvfp4kv.h -- C ABI of the NVFP4 KV cache and multi-shot sink-window
 * attention library for NVIDIA B200 (sm_100a).
 *
 * What it computes (web pages about LongLive-2.0, arXiv 2605.18739):
 *   - chunk-level NVFP4 quantization of a video DiT's KV cache, with
 *     K-smoothing and micro-block scales ("2605-LongLive2" DeepRead page,
 *     Method > 推理基础设施, parallel KV quantization; tailorednewshub page
 *     "Infrastruttura Parallela NVFP4", Inferenza W4A4 NVFP4: micro-block
 *     scaling with Four Over Six scale selection);
 *   - the Four-Over-Six block scale search over targets 6 and 4 (DeepRead
 *     page, Method > 训练基础设施, adaptive block scaling);
 *   - sliding-window self-attention with a global sink A_g and a shot sink
 *     A_s over K_eff(t) = A_g u A_s u KV[t-W, t), overlapping tokens counted
 *     once, A_s tracked by two pointers and re-bound on a prompt switch
 *     (DeepRead page, Method > 算法层设计, Multi-Shot Attention Sink).
 *   - a 3D rotary position embedding of queries and keys with the multi-shot
 *     frame offset, fused into the quantizer for K (txtmix page "LongLive 2.0：
 *     给长视频生成补上 NVFP4 并行基础设施", sections NVFP4 and 多 shot 一致性;
 *     the rotary form is a stated reading, see the rotary section below).
 *
 * Conventions for every entry point:
 *   - "device" pointers are CUDA device memory owned by the CALLER (for
 *     example torch tensors passed by data_ptr()).  The library never
 *     allocates or frees device memory and never synchronizes a stream,
 *     except nvfp4kv_workspace_status(), which synchronizes its stream.
 *   - Work is enqueued on the caller's stream and runs asynchronously.
 *     Argument errors are reported synchronously, before anything is
 *     enqueued.  Launch failures map to NVFP4KV_ERR_CUDA.  Errors found by a
 *     kernel while running (a bounded wait that gave up) are recorded in the
 *     workspace's status word and read with nvfp4kv_workspace_status().
 *   - bf16 tensors are IEEE bfloat16 bit patterns, token-major [T][H][d]
 *     (row-major, d fastest), as a video DiT lays out K, V and Q.
 *   - The CUDA kernels support head dimension d = 128 only
 *     (NVFP4KV_ERR_UNSUPPORTED otherwise).  Tensor pointers must be 16-byte
 *     aligned (NVFP4KV_ERR_ALIGNMENT).
 *   - One workspace (and one cache) per stream: calls that share one and
 *     overlap on the GPU race.
 *
 * Storage of one quantized chunk (the "rearranged, then quantized" cache of
 * the researchpapers.dev page, 推理: W4A4 加流式 VAE), head-major:
 *   k_codes, v_codes : uint8 [H][T_c][d/2]  two E2M1 codes per byte, element
 *                      2j in the low nibble of byte j (sign = bit 3)
 *   k_scales, v_scales: uint8 [H][T_c][d/16] E4M3 (fn) block scales, one per
 *                      16 consecutive channels
 *   k_mean           : float [H][d]   K-smoothing mean (added back on decode)
 *   tensor_scales    : float [2]      s_K, s_V (FP32 tensor scales)
 * Codes + block scales take (9/8)*T_c*H*d bytes against 4*T_c*H*d for bf16
 * K and V (DeepRead page, Method > 推理基础设施).
 */
#ifndef NVFP4KV_H
#define NVFP4KV_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; NULL is the legacy default stream. */
typedef struct CUstream_st* nvfp4kv_stream_t;

typedef enum {
    NVFP4KV_OK = 0,
    NVFP4KV_ERR_INVALID_ARG = 1,     /* NULL pointer, negative or zero size, ... */
    NVFP4KV_ERR_ALIGNMENT = 2,       /* a tensor pointer not 16-byte aligned */
    NVFP4KV_ERR_UNSUPPORTED = 3,     /* d != 128, or no sm_100 device */
    NVFP4KV_ERR_CAPACITY = 4,        /* too many chunks in a key set, layer out of range */
    NVFP4KV_ERR_EMPTY_KEYSET = 5,    /* attention with no key chunk */
    NVFP4KV_ERR_CUDA = 6,            /* a CUDA runtime call or launch failed */
    NVFP4KV_ERR_DEVICE_TIMEOUT = 7   /* a kernel's bounded wait gave up */
} nvfp4kv_status;

/* Element type of an output tensor. */
typedef enum {
    NVFP4KV_F32 = 0,     /* IEEE float32 */
    NVFP4KV_BF16 = 1     /* bfloat16, rounded to nearest even from float32 */
} nvfp4kv_dtype;

/* Device pointers to one quantized chunk (layouts above). */
typedef struct {
    uint8_t* k_codes;
    uint8_t* k_scales;
    uint8_t* v_codes;
    uint8_t* v_scales;
    float* k_mean;
    float* tensor_scales;
} nvfp4kv_chunk_view;

/* Largest number of chunks one attention call can read. */
#define NVFP4KV_MAX_KEY_CHUNKS 32

/* ------------------------------------------------------------------ sizes */

/* Bytes of one chunk buffer as carved by nvfp4kv_chunk_view_init: the
 * (9/8)*T_c*H*d payload, the mean, the two tensor scales, each part padded to
 * 256 bytes.  Returns 0 for invalid sizes. */
size_t nvfp4kv_chunk_bytes(int T_c, int H, int d);

/* Fill *out with the part pointers of a chunk buffer at `base` (device,
 * 256-byte aligned, nvfp4kv_chunk_bytes() long).  No device access. */
nvfp4kv_status nvfp4kv_chunk_view_init(void* base, int T_c, int H, int d,
                                       nvfp4kv_chunk_view* out);

/* Bytes of the scratch workspace the quantizer and the attention need for
 * chunks of this shape: partial sums of the K-smoothing mean, per-block
 * maxima, the grid barrier and the status word, and room for the attention's
 * partial results when it splits the key range of its last query blocks
 * (sized for up to T_c query rows; with more rows the attention runs
 * unsplit). */
size_t nvfp4kv_workspace_bytes(int T_c, int H, int d);

/* Zero the workspace's control words (status, barrier) on `stream`.  Call it
 * once after allocating a workspace, and again after a call reported
 * NVFP4KV_ERR_DEVICE_TIMEOUT. */
nvfp4kv_status nvfp4kv_workspace_init(void* ws, size_t ws_bytes, nvfp4kv_stream_t stream);

/* Synchronize `stream`, read the workspace's status word and clear it:
 * NVFP4KV_OK, NVFP4KV_ERR_DEVICE_TIMEOUT (a bounded wait inside a kernel gave
 * up), or NVFP4KV_ERR_UNSUPPORTED (an attention call met a key set whose V
 * tensor scales span more than 2^116, beyond what its fp32 softmax sums hold;
 * that call's output is not valid).  A timeout outranks the other. */
nvfp4kv_status nvfp4kv_workspace_status(void* ws, nvfp4kv_stream_t stream);

/* ------------------------------------------------------------------ quantizer */

/*
 * Quantize one frame-chunk's K and V ([T_c][H][d] bf16, device) into `out`
 * (DeepRead page, Method > 推理基础设施: chunk-level quantization,
 * K-smoothing, NVFP4 micro-blocks; Four-Over-Six per block, Method >
 * 训练基础设施).  Steps, per tensor:
 *   K only: mean[h][c] over the chunk's tokens (fp32: sums of 64-token
 *           segments, then the sum of the segments, then / T_c), and
 *           X = K - mean; for V, X = V.
 *   s = max|X| / (6*448)  (1 if the tensor is all zero).
 *   each block of 16 channels: encode with its max mapped to 6 and to 4
 *   (E4M3 block scale RNE/saturating, E2M1 codes RNE ties-to-even), keep the
 *   4-encoding only if its squared error is strictly lower.
 * Results are bit-identical to the reference definition above.
 * ws: device workspace of nvfp4kv_workspace_bytes(T_c, H, d), initialized
 * once by nvfp4kv_workspace_init.  K, V and the outputs must not overlap.
 */
nvfp4kv_status nvfp4kv_quantize_chunk(const void* K, const void* V, int T_c, int H, int d,
                                      const nvfp4kv_chunk_view* out, void* ws,
                                      nvfp4kv_stream_t stream);

/*
 * nvfp4kv_quantize_chunk without a workspace argument, for callers that are
 * not allowed to allocate device memory: an inference engine that owns every
 * byte of the GPU and gives its plugins no scratch space, or a real-time loop
 * that must not call cudaMalloc because an allocation can synchronize the
 * device and stall the other streams.  The paper has no counterpart to this
 * entry point; it is a deployment convenience.
 *
 * The scratch (partial sums, maxima, barrier and status words) lives in one
 * 4 MiB array compiled into the library, which every GPU that loads the
 * library holds until the process exits.  Chunks whose scratch,
 * 256 + ceil(T_c/64)*H*d*8 (rounded up to 256) + 32768 bytes, exceeds 4 MiB
 * are refused with NVFP4KV_ERR_CAPACITY before any device work (H = 24,
 * d = 128 allows T_c up to 10,816).  The first call on each device looks up
 * the array's device address (cudaGetSymbolAddress) with that device
 * current; make that first call before any stream capture.  The address is
 * kept for the life of the process: do not use this entry point across a
 * device reset (cudaDeviceReset, or a primary context destroyed and created
 * again), which reloads the library's module at a new address; a call that
 * fails with NVFP4KV_ERR_CUDA drops the kept address, so the next call looks
 * it up again.  Every call
 * clears the barrier and status words on `stream` and then reuses the same
 * array, so calls that overlap on the GPU (other streams, other threads)
 * race; the array keeps the last call's contents.  A kernel-side timeout is
 * not reported here; use nvfp4kv_quantize_chunk with a workspace to read it.
 * Allocates nothing: no cudaMalloc, cudaFree or allocating library routine.
 * Output, and the status returned for every argument error, are those of
 * nvfp4kv_quantize_chunk (its checks run first, in its order, the workspace
 * left out); NVFP4KV_ERR_CAPACITY follows them.
 */
nvfp4kv_status nvfp4kv_quantize_chunk_noalloc(const void* K, const void* V, int T_c, int H,
                                              int d, const nvfp4kv_chunk_view* out,
                                              nvfp4kv_stream_t stream);

/* ------------------------------------------------------------------ rotary position embedding */

/*
 * 3D rotary position embedding of a chunk's queries and keys, with the
 * multi-shot frame offset.  Source: the txtmix page "LongLive 2.0：给长视频生成
 * 补上 NVFP4 并行基础设施", section NVFP4：一条从训练贯穿到 KV cache 的量化线 (a
 * fused RoPE kernel on the NVFP4 inference path), section 多 shot 一致性
 * (inference.multi_shot_rope_offset, the RoPE position offset that keeps the
 * positions of different shots apart).  The pages give no rotary form; the
 * library implements this reading, whose parity with the pages is unpinned:
 *   - token t of a chunk lies at frame t / (rows*cols), row (t / cols) % rows,
 *     column t % cols of the latent token grid (frame-major);
 *   - the d = 128 channels of a head split into a frame part (channels
 *     0..43), a row part (44..85) and a column part (86..127); in a part of
 *     width w the channel pair (2i, 2i+1) turns by the angle
 *     p * 10000^(-2i/w), p the token's coordinate on that part's axis:
 *     (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos);
 *   - the frame coordinate is frame_pos0 + the frame within the chunk
 *     (nvfp4kv_rope_frame_position gives frame_pos0 in a multi-shot stream);
 *   - arithmetic: frequency, angle, cos and sin in double precision, cos and
 *     sin each rounded once to fp32 (nvfp4kv_rope_table); each product and
 *     sum of the rotation one fp32 rounding; results rounded to bf16.
 */

/* The geometry of one chunk's rotation. */
typedef struct {
    const void* table;   /* device, 16-byte aligned, filled by nvfp4kv_rope_table */
    int frames;          /* frames the table covers: frames * rows * cols >= T */
    int rows, cols;      /* latent tokens per frame: rows x cols */
} nvfp4kv_rope_view;

/* frame_pos0 of chunk `chunk` of a multi-shot stream: chunk * frames_per_chunk
 * frames before it, plus `offset` (multi_shot_rope_offset) once for each of
 * the `shot` shot switches before it; offset 0 counts frames as one shot.
 * Returns -1 for a negative argument or frames_per_chunk < 1.  Host only. */
long long nvfp4kv_rope_frame_position(long long chunk, int frames_per_chunk, long long shot,
                                      long long offset);

/* Bytes of a rotation table: 8 * (frames*22 + (rows + cols)*21), 0 for a
 * size outside 1 <= frames <= 2^20, rows, cols >= 1 and rows*cols <= 65535. */
size_t nvfp4kv_rope_table_bytes(int frames, int rows, int cols);

/* Fill `table` (device, 16-byte aligned, nvfp4kv_rope_table_bytes long) on
 * `stream` with float2 entries {cos, sin}: entry f*22 + i is pair i of the
 * frame part at frame coordinate frame_pos0 + f; then rows*21 entries (row r,
 * pair i at r*21 + i) and cols*21 entries (column c).  frame_pos0 in
 * [0, 2^40].  One launch. */
nvfp4kv_status nvfp4kv_rope_table(long long frame_pos0, int frames, int rows, int cols,
                                  void* table, nvfp4kv_stream_t stream);

/* Rotate X ([T][H][d] bf16, device) into Y (same layout; Y == X rotates in
 * place, other overlaps are not allowed): the queries of a chunk whose keys go
 * through nvfp4kv_quantize_chunk_rope with the same table; a partial overlap
 * is refused with NVFP4KV_ERR_INVALID_ARG.  T <= 65535,
 * T*H*H < 2^32, frames*rows*cols >= T, and the table small enough to stage in
 * shared memory: 8 * (27*frames + 26*(rows + cols)) <= 61440 bytes
 * (NVFP4KV_ERR_INVALID_ARG otherwise).  One launch; bound by HBM (2 bytes
 * read and 2 written per element). */
nvfp4kv_status nvfp4kv_rope(const void* X, void* Y, int T, int H, int d,
                            const nvfp4kv_rope_view* rope, nvfp4kv_stream_t stream);

/* nvfp4kv_quantize_chunk of (K rotated by `rope`, V): the rotation is fused
 * into the quantizer's two reads of K, so the rotated K is never stored; the
 * outputs are those of nvfp4kv_quantize_chunk on nvfp4kv_rope(K), bit for
 * bit.  The view's limits are nvfp4kv_rope's, with T = T_c. */
nvfp4kv_status nvfp4kv_quantize_chunk_rope(const void* K, const void* V, int T_c, int H,
                                           int d, const nvfp4kv_rope_view* rope,
                                           const nvfp4kv_chunk_view* out, void* ws,
                                           nvfp4kv_stream_t stream);

/* ------------------------------------------------------------------ sequence parallel */

/*
 * The chunk quantizer in three steps, for a chunk whose tokens are split over
 * several GPUs (Ulysses-style sequence parallelism: the DeepRead page, Method
 * > 推理基础设施, ships the 4-bit cache between GPUs instead of bf16).  Each
 * GPU holds one contiguous shard of the chunk's tokens, [t0, t0 + T_local),
 * for all H heads; every shard but the last starts and ends on a 64-token
 * boundary, so that the K-smoothing segments of the one-GPU definition (the
 * sequential sums over 64 tokens) fall inside one shard.  Composed as
 *   stats (each shard) -> gather the segment statistics of all shards in
 *   token order and the maximum of their max|V| -> finalize (every GPU, same
 *   result) -> encode (each shard),
 * the codes, scales, mean and tensor scales equal nvfp4kv_quantize_chunk's
 * on the whole chunk bit for bit.
 */

/* Per shard: K's per-segment column sums psum [ceil(T_local/64)][H*d] (fp32,
 * token order inside each segment), column minima / maxima pmin, pmax (same
 * shape, bf16), and max |V| over the shard (*vmax, device float).  ws: a
 * workspace of nvfp4kv_workspace_bytes(T_local, H, d). */
nvfp4kv_status nvfp4kv_chunk_stats(const void* K, const void* V, int T_local, int H, int d,
                                   float* psum, void* pmin, void* pmax, float* vmax, void* ws,
                                   nvfp4kv_stream_t stream);

/* From the statistics of all nseg = ceil(T/64) segments of the chunk (T tokens,
 * shards concatenated in token order) and the chunk's max |V|: the mean
 * k_mean [H][d] and tensor_scales {s_K, s_V}, exactly as the one-GPU
 * quantizer forms them.  ws: a workspace of nvfp4kv_workspace_bytes(1, H, d)
 * or larger. */
nvfp4kv_status nvfp4kv_chunk_finalize(const float* psum, const void* pmin, const void* pmax,
                                      int nseg, int T, int H, int d, const float* vmax,
                                      float* k_mean, float* tensor_scales, void* ws,
                                      nvfp4kv_stream_t stream);

/* Per shard: codes and block scales of its T_local tokens (out's k/v codes and
 * scales, laid out as a chunk of T_local tokens) with the chunk's k_mean and
 * tensor_scales.  out->k_mean and out->tensor_scales are not used. */
nvfp4kv_status nvfp4kv_chunk_encode(const void* K, const void* V, int T_local, int H, int d,
                                    const float* k_mean, const float* tensor_scales,
                                    const nvfp4kv_chunk_view* out, nvfp4kv_stream_t stream);

/* ------------------------------------------------------------------ head parallel */

/*
 * The chunk quantizer for a chunk whose heads are split over several GPUs:
 * each GPU holds all T tokens of its heads [h0, h1) as a [T, h1 - h0, d]
 * tensor.  The K mean and the blocks are per head; only the two tensor scales
 * couple the heads (one FP32 scale per chunk and tensor, the DeepRead page,
 * Method > 推理基础设施), and s = amax / 2688 needs the amax of the whole
 * tensor.  Composed as
 *   nvfp4kv_chunk_stats (own heads) -> nvfp4kv_chunk_amax (own heads: k_mean
 *   and the two amaxes) -> the maximum of each amax over the GPUs (one
 *   all-reduce of two floats) -> nvfp4kv_tensor_scales_from_amax ->
 *   nvfp4kv_chunk_encode (own heads),
 * each GPU's codes, scales and mean equal those heads of
 * nvfp4kv_quantize_chunk's result on the whole chunk, and every GPU's tensor
 * scales equal the whole chunk's, bit for bit.
 */

/* nvfp4kv_chunk_finalize's inputs and k_mean; instead of the tensor scales,
 * amax[0] = max |RN(K - mean)| and amax[1] = *vmax (device floats). */
nvfp4kv_status nvfp4kv_chunk_amax(const float* psum, const void* pmin, const void* pmax,
                                  int nseg, int T, int H, int d, const float* vmax,
                                  float* k_mean, float* amax, void* ws,
                                  nvfp4kv_stream_t stream);

/* tensor_scales[i] = amax[i] / 2688 (fp32, correctly rounded), or 1 where
 * amax[i] is 0; both device arrays of 2 floats. */
nvfp4kv_status nvfp4kv_tensor_scales_from_amax(const float* amax, float* tensor_scales,
                                               nvfp4kv_stream_t stream);

/* ------------------------------------------------------------------ weights / activations */

/* Block shape of nvfp4kv_quantize_matrix. */
typedef enum {
    NVFP4KV_BLOCKS_1D = 1,   /* 16 consecutive elements of a row (activations) */
    NVFP4KV_TILES_2D = 2     /* 16 x 16 tiles (weights) */
} nvfp4kv_block_shape;

/* Bytes of the workspace of nvfp4kv_quantize_matrix (any shape). */
size_t nvfp4kv_matrix_workspace_bytes(void);

/*
 * NVFP4 quantization of a weight or activation matrix with Four-Over-Six
 * (DeepRead page, Method > 训练基础设施: NVFP4 weights and activations, E2M1
 * values under FP8 E4M3 block scales and one FP32 tensor scale, each block's
 * scale searched over targets 6 and 4; the block shape follows the operand --
 * 1D for activations, 2D 16 x 16 for weights).
 *   X: [M][N] bf16 row-major, device, 16-byte aligned; N a multiple of 16
 *      (and M too for NVFP4KV_TILES_2D), else NVFP4KV_ERR_UNSUPPORTED.
 *   s = max|X| / (6*448) (1 if all zero), written to *tensor_scale (device float).
 *   Per block and target m in {6, 4}: sb = E4M3(amax / (m*s)), D = decode(sb)*s,
 *   codes E2M1(x / D) (+0 when D == 0); the block error adds, row segment by
 *   row segment in increasing row order, (e_0^2 + .. + e_7^2) + (e_8^2 + ..
 *   + e_15^2); the 4-encoding is kept only if its error is strictly lower.
 *   codes:  [M][N/2] bytes (device, 16-byte aligned), element 2j of a row in
 *           the low nibble of byte j;
 *   scales: [M][N/16] (1D) or [M/16][N/16] (2D) E4M3 bytes (device).
 *   ws: device, 256-byte aligned, nvfp4kv_matrix_workspace_bytes() long,
 *       initialized once with nvfp4kv_workspace_init (its status word reports
 *       a grid barrier that gave up, see nvfp4kv_workspace_status).
 * Results are bit-identical to the definition above.  The caller owns all
 * memory; X and the outputs must not overlap.
 */
nvfp4kv_status nvfp4kv_quantize_matrix(const void* X, int M, int N, int mode, void* codes,
                                       void* scales, float* tensor_scale, void* ws,
                                       nvfp4kv_stream_t stream);

/*
 * De-quantize a chunk back to [T_c][H][d] (device): x = decode(q) *
 * (decode(scale) * s), plus mean for K, each step one fp32 operation (the
 * DeepRead page, Method > 推理基础设施: the cache is read back through its
 * block and tensor scales, with K's mean restored).
 *   in: the chunk's device pointers (16-byte aligned, as nvfp4kv_chunk_view_init
 *       carves them); K_out, V_out: device, 16-byte aligned, T_c * H * d
 *       elements each of out_dtype, or NULL to skip that tensor.
 *   out_dtype: NVFP4KV_F32 or NVFP4KV_BF16 (the fp32 value rounded to nearest
 *       even), the same for both outputs.
 * One kernel launch for both tensors; nothing is allocated.  Errors:
 * NVFP4KV_ERR_INVALID_ARG (null view, bad shape or dtype),
 * NVFP4KV_ERR_UNSUPPORTED (d != 128, or no sm_100 device),
 * NVFP4KV_ERR_ALIGNMENT, NVFP4KV_ERR_CUDA (launch failure).  Outputs must not
 * overlap the chunk.
 */
nvfp4kv_status nvfp4kv_dequantize(const nvfp4kv_chunk_view* in, int T_c, int H, int d,
                                  void* K_out, void* V_out, int out_dtype,
                                  nvfp4kv_stream_t stream);

/* ------------------------------------------------------------------ attention */

/*
 * O = softmax(scale * Q K_hat^T) V_hat over every key of the listed chunks
 * (in any order; the caller passes the de-duplicated key set), with K_hat
 * and V_hat the de-quantized cache, non-causal inside a chunk (DeepRead page,
 * Method > 算法层设计; fused de-quantization, Method > 推理基础设施).
 *   chunks: host array of n_chunks (1..NVFP4KV_MAX_KEY_CHUNKS) views, each of
 *           T_c tokens, H heads, d = 128.
 *   Q:      [T_q][H][d] bf16, device.
 *   O:      [T_q][H][d] device, written, element type o_dtype (NVFP4KV_F32 or
 *           NVFP4KV_BF16).
 *   softmax_scale: <= 0 selects 1/sqrt(d).
 *   ws:     workspace as for the quantizer (status word only).
 * Softmax statistics are fp32; the products run on the tensor cores in fp16
 * (the de-quantized codes times their block scales are exact fp16 numbers;
 * Q is scaled by a power of two into fp16 range; s_K, the K mean and s_V
 * enter in fp32); the normalized result is stored in o_dtype.  Chunks' V
 * tensor scales may differ by up to 2^116 within one key set; a wider spread
 * is reported by nvfp4kv_workspace_status as NVFP4KV_ERR_UNSUPPORTED.
 */
nvfp4kv_status nvfp4kv_attention(const nvfp4kv_chunk_view* chunks, int n_chunks,
                                 int T_c, int H, int d, const void* Q, int T_q,
                                 void* O, int o_dtype, float softmax_scale, void* ws,
                                 nvfp4kv_stream_t stream);

/*
 * Number of kernels one attention call of this shape enqueues: 1, or 2 when
 * the query blocks left over for the GPU's last, partial wave are split
 * along the keys and merged by a second kernel (the split is an execution
 * detail: the result is the same softmax attention).  0 for invalid sizes.
 * Host-only; queries the current device's multiprocessor count once.
 */
int nvfp4kv_attention_launches(int n_chunks, int T_c, int H, int d, int T_q);

/*
 * Bytes of the caller's buffer for the NVFP4 queries of
 * nvfp4kv_attention_fp4q.  With R = T_q * H and up(x) = x rounded up to a
 * multiple of 256: E2M1 codes [R][d / 2] at offset 0 (two per byte, the even
 * element in the low nibble), E4M3 block scales [R][d / 16] at up(R d / 2),
 * the FP32 tensor scale at up(R d / 2) + up(R d / 16); total that + 256.
 * 0 for invalid sizes or d != 128.
 */
size_t nvfp4kv_fp4q_bytes(int T_q, int H, int d);

/*
 * Attention with an FP4-operand S = Q K^T (DeepRead page, Method >
 * 推理基础设施: W4A4 on Blackwell, FP4 GEMMs in place of BF16 ones): the
 * queries are quantized to NVFP4 as the activation matrix [T_q * H][d]
 * (16-element blocks along d, Four-Over-Six, one FP32 tensor scale s_Q --
 * nvfp4kv_quantize_matrix with NVFP4KV_BLOCKS_1D, Method > 训练基础设施), and
 *   S = s_Q s_K sum_blocks (q_Q sb_Q)(q_K sb_K) + Q_hat . mean
 * runs on the block-scaled FP4 tensor cores straight from the cache's E2M1
 * codes and E4M3 block scales; softmax and P V are nvfp4kv_attention's.  The
 * result is softmax attention with Q replaced by its NVFP4 reconstruction
 * Q_hat.
 *   Arguments as nvfp4kv_attention, plus
 *   q_fp4: device, 256-byte aligned, nvfp4kv_fp4q_bytes(T_q, H, d) bytes,
 *          caller-owned; written with the quantized queries (readable after
 *          the call, in the layout nvfp4kv_fp4q_bytes states).
 *   ws:    a workspace of nvfp4kv_workspace_bytes(T_c, H, d) bytes; the
 *          query quantizer uses it as its own workspace first (it is at least
 *          nvfp4kv_matrix_workspace_bytes() long).
 * Enqueues nvfp4kv_attention_fp4q_launches() kernels; allocates nothing.
 * Errors as nvfp4kv_attention (ERR_ALIGNMENT also for q_fp4); the status of
 * the device work (a wait that gave up, a V-scale spread beyond 2^116) is
 * read with nvfp4kv_workspace_status.  Q_hat . mean is taken in fp32 from the
 * decoded queries; S's block products are summed by the tensor core in fp32.
 */
nvfp4kv_status nvfp4kv_attention_fp4q(const nvfp4kv_chunk_view* chunks, int n_chunks,
                                      int T_c, int H, int d, const void* Q, int T_q,
                                      void* O, int o_dtype, float softmax_scale,
                                      void* q_fp4, void* ws, nvfp4kv_stream_t stream);

/* Kernels one nvfp4kv_attention_fp4q call enqueues: the query quantizer, the
 * attention kernel, and the merge kernel when the last wave is split (2 or
 * 3); 0 for invalid sizes.  Host-only. */
int nvfp4kv_attention_fp4q_launches(int n_chunks, int T_c, int H, int d, int T_q);

/* ------------------------------------------------------------------ cache */

/* Cache shape.  Sinks and window count whole chunks (a chunk = F_c frames of
 * T_c tokens, DeepRead page, Method > 推理基础设施): S_g global-sink chunks
 * [0, S_g), S_s shot-sink chunks from the current shot's first chunk, and the
 * W newest chunks including the one just appended. */
typedef struct {
    int layers;
    int H;
    int d;
    int T_c;
    int S_g;
    int S_s;
    int W;
} kvcache_config;

typedef struct kvcache kvcache;   /* host object; opaque */

/* Slots per layer (S_g + S_s + W, at least 1) times layers times
 * nvfp4kv_chunk_bytes(T_c, H, d). */
size_t kvcache_pool_bytes(const kvcache_config* cfg);

/*
 * Create a cache over caller-owned device memory: `pool` of
 * kvcache_pool_bytes() (256-byte aligned) and `ws` of
 * nvfp4kv_workspace_bytes(T_c, H, d).  No device access: the first
 * kvcache_append zeroes the workspace's control words on its own stream.  The
 * shot sink starts at chunk 0.  *out is a host object released with
 * kvcache_destroy.
 */
nvfp4kv_status kvcache_create(const kvcache_config* cfg, void* pool, void* ws, kvcache** out);
void kvcache_destroy(kvcache* cache);

/*
 * Append the next chunk of `layer`: chunk id n = number of chunks appended to
 * this layer so far.  Frees the slots of chunks that leave A_g u A_s u the
 * window, then quantizes K and V ([T_c][H][d] bf16, device) into a free slot
 * in place, on `stream`.  A chunk that no future attention can read (W = 0
 * and not a sink chunk) is counted but not stored.
 */
nvfp4kv_status kvcache_append(kvcache* cache, int layer, const void* K, const void* V,
                              nvfp4kv_stream_t stream);

/* kvcache_append with K rotated by `rope` (nvfp4kv_quantize_chunk_rope): the
 * cache holds the quantized rotated keys.  The table covers the chunk's
 * frames (frame_pos0 = nvfp4kv_rope_frame_position of this chunk). */
nvfp4kv_status kvcache_append_rope(kvcache* cache, int layer, const void* K, const void* V,
                                   const nvfp4kv_rope_view* rope, nvfp4kv_stream_t stream);

/*
 * Prompt switch p_k -> p_k' (DeepRead page, Method > 算法层设计): the shot
 * sink moves to [first_chunk_of_shot, first_chunk_of_shot + S_s) for every
 * layer; the global sink and the history are kept.  Call it before appending
 * that chunk.  Host bookkeeping only (two pointers, no device memory).
 * NVFP4KV_ERR_INVALID_ARG (nothing changed) if a chunk of the new sink was
 * appended to some layer already and is no longer stored there.
 */
nvfp4kv_status kvcache_rebind_shot_sink(kvcache* cache, int64_t first_chunk_of_shot);

/* The sorted, de-duplicated chunk ids `layer` attends now, written to ids
 * (room for S_g + S_s + W entries); *count receives their number. */
nvfp4kv_status kvcache_keyset(const kvcache* cache, int layer, int64_t* ids, int* count);

/* Chunks appended to `layer` so far. */
nvfp4kv_status kvcache_num_chunks(const kvcache* cache, int layer, int64_t* n);

/* Device views of a stored chunk (NVFP4KV_ERR_INVALID_ARG if not stored). */
nvfp4kv_status kvcache_chunk_view(const kvcache* cache, int layer, int64_t chunk,
                                  nvfp4kv_chunk_view* out);

/*
 * Bookkeeping half of kvcache_append without the quantization: frees slots
 * leaving the key set, claims one for the next chunk and returns its view in
 * *out (out->k_codes == NULL when the chunk is not stored).  For callers that
 * fill the slot themselves, and for host-side tests.
 */
nvfp4kv_status kvcache_advance(kvcache* cache, int layer, nvfp4kv_chunk_view* out);

/*
 * Checkpoint and resume of a cache (host bookkeeping; no device access).  A
 * checkpoint is kvcache_get_state's bytes plus a copy of the pool's
 * kvcache_pool_bytes() bytes, which the caller makes (and restores) with its
 * own copies; the workspace holds nothing that outlives a call.
 * kvcache_state_bytes: the size of the serialized state for this cache's
 * configuration: a 4-byte tag "NVKV", a uint32 format version (1), the seven
 * int32 fields of kvcache_config, the shot sink's first chunk (int64), the
 * chunks appended per layer (int64 [layers]) and the chunk id held by every
 * slot (int64 [layers][S_g + S_s + W, at least 1], -1 for a free slot), in
 * host byte order.
 * kvcache_get_state writes it into buf (host, at least kvcache_state_bytes).
 * kvcache_set_state replaces the bookkeeping of a cache created with the same
 * configuration, over a pool that holds the saved pool's bytes.  It returns
 * NVFP4KV_ERR_INVALID_ARG and changes nothing if the buffer is short or not
 * this format, the configuration differs, or the state is inconsistent (a
 * negative count or shot-sink chunk, a slot holding a chunk outside
 * [0, count), a chunk held by two slots of a layer).
 */
size_t kvcache_state_bytes(const kvcache* cache);
nvfp4kv_status kvcache_get_state(const kvcache* cache, void* buf, size_t bytes);
nvfp4kv_status kvcache_set_state(kvcache* cache, const void* buf, size_t bytes);

/*
 * Sink-window attention of `layer`'s queries Q [T_q][H][d] (bf16, device)
 * over its current key set, written to O [T_q][H][d] (device, o_dtype): the
 * key set of kvcache_keyset() passed to nvfp4kv_attention().
 * NVFP4KV_ERR_EMPTY_KEYSET if no chunk is attended.
 */
nvfp4kv_status sink_window_attention(const kvcache* cache, int layer, const void* Q, int T_q,
                                     void* O, int o_dtype, float softmax_scale,
                                     nvfp4kv_stream_t stream);

/* The cache's workspace status (see nvfp4kv_workspace_status). */
nvfp4kv_status kvcache_check_status(kvcache* cache, nvfp4kv_stream_t stream);

/* ------------------------------------------------------------------ checks */

/*
 * Element-wise use of the GPU's own format conversions, exported so that
 * tests can compare them with a reference on every input they choose:
 * op 0: E2M1 code of each fp32 input (one code per output byte),
 * op 1: E4M3 byte of each fp32 input, op 2: fp32 value of each E2M1 code,
 * op 3: fp32 value of each E4M3 byte, op 4: the fp32 quotient x/D that the
 * quantizer forms for a pair (in[2i] = x, in[2i+1] = D > 0), op 5: 2^x
 * by the attention softmax's polynomial on the FMA pipe (inputs below -125
 * are taken as -125).
 * in/out are device arrays of n elements (op 4: n quotients from 2n inputs).
 */
nvfp4kv_status nvfp4kv_check_formats(int op, const void* in, void* out, size_t n,
                                     nvfp4kv_stream_t stream);

/* Library version string. */
const char* nvfp4kv_version(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4KV_H */
