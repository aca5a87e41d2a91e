/*
 * oracle.c -- plain, slow, obviously-correct CPU reference for the NVFP4 KV
 * cache and the multi-shot sink-window attention that reads it.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the oracle that the CUDA library is
 * checked against.  Only the test suite, the smoke check and the CPU-baseline
 * leg of the benchmark may load it.  It shares no code, header, table or
 * constant generator with the CUDA library, and includes nothing from it.
 *
 * Sources (web pages about LongLive-2.0, arXiv 2605.18739):
 *   [DR]  "2605-LongLive2" DeepRead summary (kendrick-stein.github.io),
 *         Method > 训练基础设施 (NVFP4 training: E2M1 values, block FP8 E4M3
 *         scale, tensor FP32 scale; scale search over targets 6 and 4),
 *         Method > 推理基础设施 (parallel KV quantization: chunk level,
 *         K-smoothing, micro-block NVFP4, (9/8)T_c*H*d bytes; W4A4 on
 *         Blackwell, FP4 GEMMs in place of BF16 ones -- the attention over
 *         fp32 queries serves the FP4-query form of S = Q K^T),
 *         Method > 算法层设计 (Multi-Shot Attention Sink: A_g, A_s,
 *         K_eff(t) = A_g u A_s u KV[t-W,t), de-duplication, two pointers).
 *   [TN]  "LongLive-2.0: Infrastruttura Parallela NVFP4 per Video Lunghi"
 *         (tailorednewshub), Infrastruttura di Inferenza > Inferenza W4A4
 *         NVFP4 (micro-block scaling, Four Over Six on the KV cache).
 *   [RP]  "LongLive-2.0:用 NVFP4 4 比特训练与推理长视频" (researchpapers.dev),
 *         推理:W4A4 加流式 VAE (KV rearranged, then quantized per micro-block).
 *
 * Where the pages leave a step open, the reading taken is the plainest one
 * the rest supports, restated at the function that implements it:
 *   - micro-block = 16 contiguous channels along d;
 *   - E2M1 magnitudes {0, .5, 1, 1.5, 2, 3, 4, 6}, round to nearest, ties to
 *     the even code, saturate at 6, sign copied from the input;
 *   - E4M3 = the "fn" variant (bias 7, max 448, no infinities), round to
 *     nearest even, saturate at 448, subnormals kept;
 *   - one FP32 tensor scale per chunk and per K/V: s = amax / (6 * 448);
 *   - Four-Over-Six: encode each block with its max mapped to 6 and to 4 and
 *     keep 4 only if its squared error is strictly lower;
 *   - K-smoothing: per-head, per-channel mean of K over the chunk's tokens,
 *     fp32, summed in 64-token segments (the canonical order below);
 *   - sinks and window in whole chunks; window = the W newest chunks
 *     including the one just appended.
 *
 * Floating point: every fp32 step below is a single IEEE operation rounded to
 * nearest even.  The file is compiled with -ffp-contract=off and without
 * fast-math so that no multiply-add is fused and no step is reassociated.
 * Attention is computed in double precision.
 */
#include <math.h>
#include <omp.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* bf16                                                                     */
/* ------------------------------------------------------------------------ */

/* bf16 is the top half of an IEEE binary32: widening is exact. */
float oracle_bf16_to_f32(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* Round an fp32 value to bf16, nearest even (NaN is not expected here). */
uint16_t oracle_f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* E2M1 (4-bit element) -- [DR] Method > 训练基础设施 names E2M1 values.     */
/* Code layout: bit 3 = sign, bits 2..0 = magnitude index into             */
/* {0, 0.5, 1, 1.5, 2, 3, 4, 6}.                                            */
/* ------------------------------------------------------------------------ */

static const float E2M1_MAGNITUDE[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float oracle_e2m1_decode(uint8_t code) {
    float m = E2M1_MAGNITUDE[code & 7u];
    return (code & 8u) ? -m : m;
}

/*
 * Nearest grid magnitude, ties to the even code, saturating at 6.  The sign
 * bit is copied from y even when the magnitude rounds to zero, so -0 codes
 * (0x8) occur.  Written as the list of decision points between neighbouring
 * grid values; at a decision point exactly, the neighbour with the even
 * magnitude index wins.
 */
uint8_t oracle_e2m1_encode(float y) {
    uint8_t sign = signbit(y) ? 8u : 0u;
    float a = fabsf(y);
    uint8_t idx;
    if (a < 0.25f)       idx = 0;
    else if (a == 0.25f) idx = 0;   /* tie 0 | 0.5  -> index 0 (even) */
    else if (a < 0.75f)  idx = 1;
    else if (a == 0.75f) idx = 2;   /* tie 0.5 | 1  -> index 2 */
    else if (a < 1.25f)  idx = 2;
    else if (a == 1.25f) idx = 2;   /* tie 1 | 1.5  -> index 2 */
    else if (a < 1.75f)  idx = 3;
    else if (a == 1.75f) idx = 4;   /* tie 1.5 | 2  -> index 4 */
    else if (a < 2.5f)   idx = 4;
    else if (a == 2.5f)  idx = 4;   /* tie 2 | 3    -> index 4 */
    else if (a < 3.5f)   idx = 5;
    else if (a == 3.5f)  idx = 6;   /* tie 3 | 4    -> index 6 */
    else if (a < 5.0f)   idx = 6;
    else if (a == 5.0f)  idx = 6;   /* tie 4 | 6    -> index 6 */
    else                 idx = 7;   /* above 5, saturating at 6 */
    return (uint8_t)(sign | idx);
}

/* ------------------------------------------------------------------------ */
/* E4M3 "fn" (8-bit block scale) -- [DR] Method > 训练基础设施: block-wise   */
/* FP8 E4M3.  Bias 7, no infinities, 0x7F/0xFF are NaN, max finite 448.     */
/* ------------------------------------------------------------------------ */

float oracle_e4m3_decode(uint8_t b) {
    int s = (b >> 7) & 1;
    int e = (b >> 3) & 15;
    int m = b & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0) v = ldexp((double)m, -9);                    /* m/8 * 2^-6 */
    else        v = ldexp(1.0 + (double)m / 8.0, e - 7);
    return (float)(s ? -v : v);                             /* exact */
}

/*
 * Round a non-negative finite fp32 value to E4M3, nearest even, saturating
 * at 448, keeping subnormals (spacing 2^-9 below 2^-6).  Negative inputs do
 * not occur in the quantizer (block maxima are magnitudes); they are encoded
 * through their magnitude with the sign bit set.
 */
uint8_t oracle_e4m3_encode(float y) {
    uint8_t sign = signbit(y) ? 0x80u : 0u;
    double a = fabs((double)y);                 /* exact widening */
    if (a >= 448.0) return (uint8_t)(sign | 0x7Eu);   /* satfinite: 448 */
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: value = k * 2^-9, k = RNE(a * 2^9), k in 0..8 */
        double k = nearbyint(ldexp(a, 9));      /* default mode: ties-to-even */
        /* k == 8 is the smallest normal 2^-6 = exponent 1, mantissa 0 */
        return (uint8_t)(sign | (uint8_t)k);    /* 8 == 0b0001000 */
    }
    int e;
    double fr = frexp(a, &e);                   /* a = fr * 2^e, fr in [0.5,1) */
    int E = e - 1;                              /* a = (2*fr) * 2^E, 2*fr in [1,2) */
    double mant = nearbyint((2.0 * fr - 1.0) * 8.0);  /* 3 mantissa bits, RNE */
    if (mant == 8.0) { mant = 0.0; E += 1; }
    int field = E + 7;
    uint8_t code = (uint8_t)((field << 3) | (int)mant);
    if (code > 0x7Eu) code = 0x7Eu;            /* rounding up past 448 saturates */
    return (uint8_t)(sign | code);
}

/* ------------------------------------------------------------------------ */
/* Chunk quantization -- [DR] Method > 推理基础设施; [TN] Inferenza W4A4.    */
/* ------------------------------------------------------------------------ */

#define SEGMENT_TOKENS 64       /* K-smoothing partial-sum segment length */
#define BLOCK 16                /* micro-block length along d            */
#define TENSOR_SCALE_DIV 2688.0f  /* 6 * 448: the largest E2M1 x largest E4M3 */

/*
 * K-smoothing mean, per head and channel (K only).  Canonical fp32 order:
 * sequential sum inside each 64-token segment in increasing t, then a
 * sequential sum of the segment sums in increasing segment index, then one
 * IEEE division by T.  X is [T][H][d] bf16.  mean is [H][d].
 */
void oracle_k_mean(const uint16_t* X, int T, int H, int d, float* mean) {
    int nseg = (T + SEGMENT_TOKENS - 1) / SEGMENT_TOKENS;
    #pragma omp parallel for schedule(static)
    for (int h = 0; h < H; ++h) {
        for (int c = 0; c < d; ++c) {
            float S = 0.0f;
            for (int s = 0; s < nseg; ++s) {
                int t0 = s * SEGMENT_TOKENS;
                int t1 = t0 + SEGMENT_TOKENS < T ? t0 + SEGMENT_TOKENS : T;
                float P = 0.0f;
                for (int t = t0; t < t1; ++t)
                    P = P + oracle_bf16_to_f32(X[((size_t)t * H + h) * d + c]);
                S = S + P;
            }
            mean[h * d + c] = S / (float)T;
        }
    }
}

/*
 * Encode one 16-element block x[0..15] for one target magnitude m (6 or 4):
 * block scale byte, 16 codes, and the block's squared error.
 *   sb = E4M3(a_b / (m*s)),  D = decode(sb) * s,
 *   q_i = E2M1(x_i / D) (or +0 when D == 0),
 *   e_i = x_i - decode(q_i)*D,
 *   E = (e_0^2 + ... + e_7^2) + (e_8^2 + ... + e_15^2), each half summed
 *       left to right.
 */
static void encode_block_target(const float* x, float amax, float s, float m,
                                uint8_t* sb_out, uint8_t* q, float* err_out) {
    float ms = m * s;
    float ratio = amax / ms;
    uint8_t sb = oracle_e4m3_encode(ratio);
    float D = oracle_e4m3_decode(sb) * s;
    for (int i = 0; i < BLOCK; ++i) {
        if (D > 0.0f) {
            float y = x[i] / D;
            q[i] = oracle_e2m1_encode(y);
        } else {
            q[i] = 0;
        }
    }
    float lo = 0.0f, hi = 0.0f;
    for (int i = 0; i < BLOCK; ++i) {
        float recon = oracle_e2m1_decode(q[i]) * D;
        float e = x[i] - recon;
        float e2 = e * e;
        if (i < BLOCK / 2) lo = (i == 0) ? e2 : lo + e2;
        else               hi = (i == BLOCK / 2) ? e2 : hi + e2;
    }
    *sb_out = sb;
    *err_out = lo + hi;
}

/*
 * Quantize one tensor of one chunk.  X: [T][H][d] bf16 (host).  If mean is
 * non-NULL the tensor is K: its K-smoothing mean is computed into mean[H][d]
 * and subtracted first.  Outputs (head-major, the "rearranged" layout of
 * [RP] 推理): codes [H][T][d/2] (element 2j in the low nibble of byte j),
 * scales [H][T][d/16] (E4M3 bytes), *tensor_scale, and optionally
 * choice [H][T][d/16] (1 where target 4 was kept, else 0).
 */
void oracle_quantize_tensor(const uint16_t* X, int T, int H, int d, float* mean,
                            uint8_t* codes, uint8_t* scales, float* tensor_scale,
                            uint8_t* choice) {
    size_t n = (size_t)T * H * d;
    float* Xs = (float*)malloc(n * sizeof(float));
    if (mean) oracle_k_mean(X, T, H, d, mean);

    /* X' = X - mean (K) or X (V); A = max |X'| over the tensor */
    float A = 0.0f;
    #pragma omp parallel for schedule(static) reduction(max:A)
    for (int t = 0; t < T; ++t)
        for (int h = 0; h < H; ++h)
            for (int c = 0; c < d; ++c) {
                size_t i = ((size_t)t * H + h) * d + c;
                float v = oracle_bf16_to_f32(X[i]);
                if (mean) v = v - mean[h * d + c];
                Xs[i] = v;
                float av = fabsf(v);
                if (av > A) A = av;
            }
    float s = (A > 0.0f) ? A / TENSOR_SCALE_DIV : 1.0f;
    *tensor_scale = s;

    int nb = d / BLOCK;
    #pragma omp parallel for schedule(static)
    for (int h = 0; h < H; ++h)
        for (int t = 0; t < T; ++t)
            for (int b = 0; b < nb; ++b) {
                const float* x = Xs + ((size_t)t * H + h) * d + b * BLOCK;
                float amax = 0.0f;
                for (int i = 0; i < BLOCK; ++i) {
                    float av = fabsf(x[i]);
                    if (av > amax) amax = av;
                }
                uint8_t sb6, sb4, q6[BLOCK], q4[BLOCK];
                float e6, e4;
                encode_block_target(x, amax, s, 6.0f, &sb6, q6, &e6);
                encode_block_target(x, amax, s, 4.0f, &sb4, q4, &e4);
                int keep4 = e4 < e6;            /* a tie keeps target 6 */
                const uint8_t* q = keep4 ? q4 : q6;
                size_t row = (size_t)h * T + t;
                scales[row * nb + b] = keep4 ? sb4 : sb6;
                if (choice) choice[row * nb + b] = (uint8_t)keep4;
                uint8_t* out = codes + row * (d / 2) + b * (BLOCK / 2);
                for (int j = 0; j < BLOCK / 2; ++j)
                    out[j] = (uint8_t)((q[2 * j] & 15u) | ((q[2 * j + 1] & 15u) << 4));
            }
    free(Xs);
}

/*
 * NVFP4 quantization of a weight or activation matrix with Four-Over-Six
 * ([DR] Method > 训练基础设施: NVFP4 weights and activations -- E2M1 values,
 * FP8 E4M3 block scales, an FP32 tensor scale, the block scale searched over
 * targets 6 and 4; the block shape follows the operand: 1D blocks along a row
 * for activations, 2D 16 x 16 blocks for weights).
 *   X: [M][N] bf16, row-major; N a multiple of 16 (and M too for 2D).
 *   mode 1 (activations): a block is 16 consecutive elements of a row;
 *          scales [M][N/16].
 *   mode 2 (weights): a block is a 16 x 16 tile; scales [M/16][N/16].
 *   s = max|X| / (6*448)  (1 if X is all zero).
 * Per block and target m: sb = E4M3(amax / (m*s)), D = decode(sb) * s,
 * q_i = E2M1(x_i / D) (+0 when D == 0), e_i = x_i - decode(q_i)*D.  The block
 * error, in fp32: each 16-element row segment of the block gives
 * (e_0^2 + .. + e_7^2) + (e_8^2 + .. + e_15^2) (each half left to right), and
 * the segments are added in increasing row order -- the same as the KV blocks
 * for 1D.  Keep 4 only if its error is strictly lower.
 * Codes [M][N/2], element 2j of a row in the low nibble of byte j.
 * choice (optional): [number of blocks], 1 where target 4 was kept.
 * Returns 0, or -1 for shapes the mode does not tile.
 */
static float matrix_segment(const float* x, float D, uint8_t* q) {
    float lo = 0.0f, hi = 0.0f;
    for (int i = 0; i < BLOCK; ++i) {
        q[i] = (D > 0.0f) ? oracle_e2m1_encode(x[i] / D) : 0;
        float e = x[i] - oracle_e2m1_decode(q[i]) * D;
        float e2 = e * e;
        if (i < BLOCK / 2) lo = (i == 0) ? e2 : lo + e2;
        else               hi = (i == BLOCK / 2) ? e2 : hi + e2;
    }
    return lo + hi;
}

int oracle_quantize_matrix(const uint16_t* X, int M, int N, int mode, uint8_t* codes,
                           uint8_t* scales, float* tensor_scale, uint8_t* choice) {
    if (M <= 0 || N <= 0 || N % BLOCK != 0 || (mode == 2 && M % BLOCK != 0) ||
        (mode != 1 && mode != 2))
        return -1;
    size_t n = (size_t)M * N;
    float* Xf = (float*)malloc(n * sizeof(float));
    float A = 0.0f;
    #pragma omp parallel for schedule(static) reduction(max:A)
    for (long long i = 0; i < (long long)n; ++i) {
        Xf[i] = oracle_bf16_to_f32(X[i]);
        float av = fabsf(Xf[i]);
        if (av > A) A = av;
    }
    float s = (A > 0.0f) ? A / TENSOR_SCALE_DIV : 1.0f;
    *tensor_scale = s;
    const int rows = (mode == 1) ? 1 : BLOCK;            /* row segments per block */
    const int brows = M / rows, bcols = N / BLOCK;
    #pragma omp parallel for schedule(static)
    for (int br = 0; br < brows; ++br)
        for (int bc = 0; bc < bcols; ++bc) {
            float amax = 0.0f;
            for (int r = 0; r < rows; ++r)
                for (int i = 0; i < BLOCK; ++i) {
                    float av = fabsf(Xf[(size_t)(br * rows + r) * N + bc * BLOCK + i]);
                    if (av > amax) amax = av;
                }
            uint8_t sb[2], q[2][BLOCK * BLOCK];
            float err[2];
            const float targets[2] = {6.0f, 4.0f};
            for (int k = 0; k < 2; ++k) {
                float ratio = amax / (targets[k] * s);
                sb[k] = oracle_e4m3_encode(ratio);
                float D = oracle_e4m3_decode(sb[k]) * s;
                float E = 0.0f;
                for (int r = 0; r < rows; ++r) {
                    float seg = matrix_segment(Xf + (size_t)(br * rows + r) * N + bc * BLOCK, D,
                                               q[k] + r * BLOCK);
                    E = (r == 0) ? seg : E + seg;
                }
                err[k] = E;
            }
            int keep4 = err[1] < err[0];            /* a tie keeps target 6 */
            scales[(size_t)br * bcols + bc] = sb[keep4];
            if (choice) choice[(size_t)br * bcols + bc] = (uint8_t)keep4;
            for (int r = 0; r < rows; ++r) {
                uint8_t* out = codes + (size_t)(br * rows + r) * (N / 2) + bc * (BLOCK / 2);
                const uint8_t* qq = q[keep4] + r * BLOCK;
                for (int j = 0; j < BLOCK / 2; ++j)
                    out[j] = (uint8_t)((qq[2 * j] & 15u) | ((qq[2 * j + 1] & 15u) << 4));
            }
        }
    free(Xf);
    return 0;
}

/* De-quantize a matrix quantized by oracle_quantize_matrix: fp32 [M][N],
 * x_hat = decode(q) * (decode(sb) * s). */
void oracle_dequantize_matrix(const uint8_t* codes, const uint8_t* scales, float s, int M,
                              int N, int mode, float* out) {
    const int rows = (mode == 1) ? 1 : BLOCK;
    for (int r = 0; r < M; ++r)
        for (int c = 0; c < N; ++c) {
            uint8_t byte = codes[(size_t)r * (N / 2) + c / 2];
            uint8_t q = (c & 1) ? (byte >> 4) : (byte & 15u);
            float D = oracle_e4m3_decode(scales[(size_t)(r / rows) * (N / BLOCK) + c / BLOCK]) * s;
            out[(size_t)r * N + c] = oracle_e2m1_decode(q) * D;
        }
}

/* Both tensors of a chunk: K with smoothing, V without. */
void oracle_quantize_chunk(const uint16_t* K, const uint16_t* V, int T, int H, int d,
                           uint8_t* k_codes, uint8_t* k_scales,
                           uint8_t* v_codes, uint8_t* v_scales,
                           float* k_mean, float* tensor_scales /* [2]: s_K, s_V */) {
    oracle_quantize_tensor(K, T, H, d, k_mean, k_codes, k_scales, &tensor_scales[0], NULL);
    oracle_quantize_tensor(V, T, H, d, NULL, v_codes, v_scales, &tensor_scales[1], NULL);
}

/*
 * Dequantize one tensor back to fp32 [T][H][d]:
 *   x_hat = decode(q) * (decode(sb) * s), then + mean for K.
 */
void oracle_dequantize_tensor(const uint8_t* codes, const uint8_t* scales,
                              const float* mean, float s, int T, int H, int d,
                              float* out) {
    int nb = d / BLOCK;
    for (int h = 0; h < H; ++h)
        for (int t = 0; t < T; ++t)
            for (int c = 0; c < d; ++c) {
                size_t row = (size_t)h * T + t;
                uint8_t byte = codes[row * (d / 2) + c / 2];
                uint8_t q = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
                float D = oracle_e4m3_decode(scales[row * nb + c / BLOCK]) * s;
                float v = oracle_e2m1_decode(q) * D;
                if (mean) v = v + mean[h * d + c];
                out[((size_t)t * H + h) * d + c] = v;
            }
}

/* ------------------------------------------------------------------------ */
/* Key set -- [DR] Method > 算法层设计 (Multi-Shot Attention Sink).          */
/* ------------------------------------------------------------------------ */

/*
 * Chunk ids attended when n chunks are in the cache (the newest, n-1, was
 * just appended):
 *   A_g    = [0, S_g)                      (global sink, never evicted)
 *   A_s    = [s_begin, s_begin+S_s) n [0,n) (shot sink, two pointers)
 *   window = [max(0, n-W), n)
 * Returns their sorted union (duplicates removed) in ids; returns the count.
 * ids must hold S_g + S_s + W entries.
 */
int oracle_keyset(int64_t n, int S_g, int S_s, int W, int64_t s_begin, int64_t* ids) {
    int count = 0;
    for (int64_t c = 0; c < n; ++c) {
        int in_g = c < S_g;
        int in_s = c >= s_begin && c < s_begin + S_s;
        int in_w = c >= n - W;
        if (in_g || in_s || in_w) ids[count++] = c;
    }
    return count;
}

/* ------------------------------------------------------------------------ */
/* Attention over the de-quantized key set, in double precision.            */
/* ------------------------------------------------------------------------ */

typedef struct {
    const uint8_t* k_codes;   /* [H][T][d/2] */
    const uint8_t* k_scales;  /* [H][T][d/16] */
    const float* k_mean;      /* [H][d] */
    const uint8_t* v_codes;
    const uint8_t* v_scales;
    float s_k;
    float s_v;
    int T;
} oracle_chunk;

/* Exact double value of one stored element: decode(q)*decode(sb)*s (+mean). */
static double dq_elem(const uint8_t* codes, const uint8_t* scales, const float* mean,
                      float s, int T, int d, int h, int t, int c) {
    size_t row = (size_t)h * T + t;
    uint8_t byte = codes[row * (d / 2) + c / 2];
    uint8_t q = (c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 15u);
    double v = (double)oracle_e2m1_decode(q) *
               (double)oracle_e4m3_decode(scales[row * (d / BLOCK) + c / BLOCK]) * (double)s;
    if (mean) v += (double)mean[h * d + c];
    return v;
}

/*
 * O_i = sum_j softmax_j(scale * Q_i . K_hat_j) V_hat_j over every key of
 * every listed chunk (the caller passes the de-duplicated key set; passing a
 * chunk twice counts its keys twice).  Non-causal inside the chunk, no
 * positional encoding, the same H for queries and keys.  The softmax is the
 * textbook one, shifted by the row maximum for range.
 *   Q:    [T_q][H][d] bf16
 *   rows: query rows to evaluate (NULL = all T_q rows), n_rows of them
 *   out:  [n_rows][H][d] double
 * Loops heads outermost; keys of one head are expanded to double once.
 */
/* The attention of either Q form: Qb (bf16 bits) or Qf (fp32 values), the
 * other NULL; both are widened exactly to float64. */
static void attention_core(const oracle_chunk* chunks, int n_chunks, int H, int d,
                           const uint16_t* Qb, const float* Qf, int T_q, const int* rows,
                           int n_rows, double scale, double* out) {
    int L = 0;
    for (int k = 0; k < n_chunks; ++k) L += chunks[k].T;
    if (L == 0) return;
    if (!(scale > 0.0)) scale = 1.0 / sqrt((double)d);
    double* Kh = (double*)malloc((size_t)L * d * sizeof(double));
    double* Vh = (double*)malloc((size_t)L * d * sizeof(double));
    for (int h = 0; h < H; ++h) {
        int j = 0;
        for (int k = 0; k < n_chunks; ++k) {
            const oracle_chunk* ch = &chunks[k];
            for (int t = 0; t < ch->T; ++t, ++j)
                for (int c = 0; c < d; ++c) {
                    Kh[(size_t)j * d + c] = dq_elem(ch->k_codes, ch->k_scales, ch->k_mean,
                                                    ch->s_k, ch->T, d, h, t, c);
                    Vh[(size_t)j * d + c] = dq_elem(ch->v_codes, ch->v_scales, NULL,
                                                    ch->s_v, ch->T, d, h, t, c);
                }
        }
        #pragma omp parallel for schedule(dynamic, 1)
        for (int r = 0; r < n_rows; ++r) {
            int i = rows ? rows[r] : r;
            double* q = (double*)malloc((size_t)d * sizeof(double));
            double* p = (double*)malloc((size_t)L * sizeof(double));
            for (int c = 0; c < d; ++c) {
                const size_t e = ((size_t)i * H + h) * d + c;
                q[c] = Qb ? (double)oracle_bf16_to_f32(Qb[e]) : (double)Qf[e];
            }
            double mx = -INFINITY;
            for (int jj = 0; jj < L; ++jj) {
                double acc = 0.0;
                for (int c = 0; c < d; ++c) acc += q[c] * Kh[(size_t)jj * d + c];
                p[jj] = acc * scale;
                if (p[jj] > mx) mx = p[jj];
            }
            double sum = 0.0;
            for (int jj = 0; jj < L; ++jj) {
                p[jj] = exp(p[jj] - mx);
                sum += p[jj];
            }
            double* o = out + ((size_t)r * H + h) * d;
            for (int c = 0; c < d; ++c) o[c] = 0.0;
            for (int jj = 0; jj < L; ++jj) {
                double w = p[jj] / sum;
                for (int c = 0; c < d; ++c) o[c] += w * Vh[(size_t)jj * d + c];
            }
            free(q);
            free(p);
        }
    }
    free(Kh);
    free(Vh);
}

/* Storage of one quantized chunk (codes + block scales, K and V), bytes. */
size_t oracle_chunk_payload_bytes(int T, int H, int d) {
    size_t n = (size_t)T * H * d;
    return 2 * (n / 2 + n / BLOCK);
}

/* ------------------------------------------------------------------------ */
/* Array helpers for the test harness (loops over the scalar functions).     */
/* ------------------------------------------------------------------------ */

void oracle_attention_f64(const oracle_chunk* chunks, int n_chunks, int H, int d,
                          const uint16_t* Q, int T_q, const int* rows, int n_rows,
                          double scale, double* out) {
    attention_core(chunks, n_chunks, H, d, Q, NULL, T_q, rows, n_rows, scale, out);
}

/* The same attention for queries given as fp32 values: used with Q replaced by
 * its NVFP4 reconstruction, the FP4-operand form of S = Q K^T ("2605-LongLive2"
 * DeepRead page, Method > 推理基础设施: on Blackwell the generator runs W4A4,
 * FP4 GEMMs in place of BF16 ones; Method > 训练基础设施: activations take 1D
 * blocks along the contraction). */
void oracle_attention_f64_fq(const oracle_chunk* chunks, int n_chunks, int H, int d,
                             const float* Qf, int T_q, const int* rows, int n_rows,
                             double scale, double* out) {
    attention_core(chunks, n_chunks, H, d, NULL, Qf, T_q, rows, n_rows, scale, out);
}

/* ------------------------------------------------------------------------ */
/* Rotary position embedding of a chunk's queries or keys (a reading)       */
/* ------------------------------------------------------------------------ */

/*
 * [TX] "LongLive 2.0：给长视频生成补上 NVFP4 并行基础设施" (txtmix): the section
 * NVFP4：一条从训练贯穿到 KV cache 的量化线 names a fused RoPE kernel on the
 * NVFP4 inference path, and 多 shot 一致性 names the inference option
 * multi_shot_rope_offset, a RoPE position offset for multi-shot generation that
 * keeps the positions of different shots apart.  Neither gives the rotary form.
 * The reading taken (parity against the pages is unpinned; the tests pin this
 * function to the properties of a rotation and to closed-form values):
 *   - the latent tokens of a chunk form frames of rows x cols tokens, frame-major,
 *     then row, then column: token t is at frame t / (rows*cols), row
 *     (t / cols) % rows, column t % cols;
 *   - the d channels of a head split into three contiguous parts, one per axis:
 *     frame w0 = d - 4*(d/6) channels, row w1 = 2*(d/6), column w2 = 2*(d/6)
 *     (44, 42, 42 for d = 128);
 *   - in a part of width w, channels (2i, 2i+1) turn by the angle
 *     p * 10000^(-2i/w), p the token's coordinate on that part's axis:
 *     (x0, x1) -> (x0 cos - x1 sin, x0 sin + x1 cos);
 *   - the frame coordinate is frame_pos0 + the frame within the chunk; a
 *     multi-shot stream gives chunk n of shot s (s shot switches before it)
 *     frame_pos0 = n * frames_per_chunk + s * offset, offset being
 *     multi_shot_rope_offset (0: plain frame counting);
 *   - arithmetic: the frequency, the angle, cos and sin in double precision;
 *     cos and sin each rounded once to fp32; each of the four products and the
 *     two sums one fp32 rounding; the two results rounded to bf16 (the model's
 *     queries and keys are bf16).
 * Y may be X (each channel pair is read before it is written).
 */
void oracle_rope_cos_sin(int64_t p, int i, int w, float* c, float* s) {
    const double omega = pow(10000.0, (double)(-2 * i) / (double)w);
    const double phi = (double)p * omega;
    *c = (float)cos(phi);
    *s = (float)sin(phi);
}

void oracle_rope(const uint16_t* X, int T, int H, int d, int64_t frame_pos0, int rows,
                 int cols, uint16_t* Y) {
    const int w[3] = {d - 4 * (d / 6), 2 * (d / 6), 2 * (d / 6)};
    for (int t = 0; t < T; ++t) {
        const int64_t pos[3] = {frame_pos0 + t / (rows * cols), (t / cols) % rows, t % cols};
        for (int h = 0; h < H; ++h) {
            const uint16_t* x = X + ((size_t)t * H + h) * d;
            uint16_t* y = Y + ((size_t)t * H + h) * d;
            int base = 0;
            for (int a = 0; a < 3; ++a) {
                for (int i = 0; i < w[a] / 2; ++i) {
                    float c, s;
                    oracle_rope_cos_sin(pos[a], i, w[a], &c, &s);
                    const float x0 = oracle_bf16_to_f32(x[base + 2 * i]);
                    const float x1 = oracle_bf16_to_f32(x[base + 2 * i + 1]);
                    const float x0c = x0 * c, x1s = x1 * s;
                    const float x0s = x0 * s, x1c = x1 * c;
                    y[base + 2 * i] = oracle_f32_to_bf16(x0c - x1s);
                    y[base + 2 * i + 1] = oracle_f32_to_bf16(x0s + x1c);
                }
                base += w[a];
            }
        }
    }
}

void oracle_set_threads(int n) { omp_set_num_threads(n > 0 ? n : 1); }
int oracle_get_threads(void) { return omp_get_max_threads(); }

void oracle_e2m1_encode_array(const float* y, uint8_t* out, size_t n) {
    for (size_t i = 0; i < n; ++i) out[i] = oracle_e2m1_encode(y[i]);
}
void oracle_e2m1_decode_array(const uint8_t* q, float* out, size_t n) {
    for (size_t i = 0; i < n; ++i) out[i] = oracle_e2m1_decode(q[i]);
}
void oracle_e4m3_encode_array(const float* y, uint8_t* out, size_t n) {
    for (size_t i = 0; i < n; ++i) out[i] = oracle_e4m3_encode(y[i]);
}
void oracle_e4m3_decode_array(const uint8_t* b, float* out, size_t n) {
    for (size_t i = 0; i < n; ++i) out[i] = oracle_e4m3_decode(b[i]);
}
void oracle_f32_to_bf16_array(const float* x, uint16_t* out, size_t n) {
    for (size_t i = 0; i < n; ++i) out[i] = oracle_f32_to_bf16(x[i]);
}
