/*
 * Plain CPU oracle for the fused W8A8 block-scaled MoE expert computation.
 *
 * TEST INFRASTRUCTURE ONLY.  This file is the slow, obviously correct
 * definition that the CUDA library is checked against.  It shares no code,
 * header, table or constant with the CUDA library and must never be linked
 * into it.  Only the tests, the smoke check and the benchmark's CPU-baseline
 * leg may load it.
 *
 * Sources (web pages that describe the method; cited by title and section):
 *  [AlphaMoE]  "FlashInfer: Blackwell W8A8 AlphaMoE Expert ..." (flashinfer
 *              PR #4287): the five-stage expert pipeline (section
 *              "문제점: MoE Expert 계산의 병목", stages 1-5), W8A8 with FP8 tensor
 *              cores ("2. W8A8 양자화 및 Blackwell Tensor Cores 활용").
 *  [Wave]      "FlashInfer SM120 MoE GEMM 최적화: 웨이브+잔여물 비용 모델 도입"
 *              (flashinfer PR #4318), "코드 분석 1.": the grouped "nt" GEMM
 *              interface with m_indptr, per-block fp32 scales with explicit
 *              (m,n,k) granularities, and the gated (gate+up, even N) form.
 *  [Cake-act]  "NVIDIA R200(SM107)을 위한 SwiGLU + MXFP8 커널 최적화"
 *              (flashinfer PR #8023): SwiGLU followed by MXFP8 quantisation;
 *              "2. build.json": IEEE divide/sqrt and no flush-to-zero.
 *
 * Arithmetic is fp32 with every operation rounded on its own
 * (build with -ffp-contract=off), no flush-to-zero, IEEE division.
 * Readings of points the pages leave open:
 *  - FP8 is OCP E4M3 "FN": bias 7, no infinities, max 448, NaN = S.1111.111.
 *  - Block scale = amax / 448 (fp32 IEEE divide); code = RNE_sat(v / scale).
 *    An all-zero block gets scale 1.0 and all codes +0.
 *  - Activations: one scale per token per 128 columns; weights: one scale per
 *    128x128 block.  The intermediate is kept in fp32 before requantisation.
 *  - w13 holds gate rows [0, I) then up rows [I, 2I); SwiGLU = silu(gate)*up.
 *  - The grouped GEMM sums each 128-wide K block in fp32 in ascending k, then
 *    multiplies the block sum by (a_scale * b_scale) and adds it to an fp32
 *    accumulator in ascending block order.
 *  - The router weight is applied after the down projection, inside the
 *    combine; the combine sums the top-k slots in ascending slot order.
 *  - Grouping is a stable counting sort of pair ids p = t*k + j by expert.
 *  - MXFP8: E8M0 scale X = 2^s with s the smallest integer such that
 *    amax <= 448 * 2^s (code s+127 clamped to [0,254]); q = RNE_sat(v / X).
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------ */
/* FP8 E4M3 (FN) and E8M0 codecs                                         */
/* ------------------------------------------------------------------ */

/* Decode one E4M3 code from its bit fields. */
float oracle_e4m3_decode(uint8_t c) {
    int sign = (c >> 7) & 1;
    int e = (c >> 3) & 15;
    int m = c & 7;
    double v;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        v = ldexp((double)m, -9);              /* subnormal: m * 2^-9 */
    else
        v = ldexp(1.0 + m / 8.0, e - 7);       /* normal: 1.m * 2^(e-7) */
    return (float)(sign ? -v : v);
}

/* Encode an fp32 value to E4M3 with round-to-nearest-even; finite values
 * whose rounded magnitude exceeds 448 saturate to 448. */
uint8_t oracle_e4m3_encode(float v) {
    if (isnan(v)) return 0x7F;
    uint8_t sign = signbit(v) ? 0x80 : 0x00;
    double a = fabs((double)v);
    if (a > 448.0) return sign | 0x7E;
    if (a < ldexp(1.0, -6)) {
        /* subnormal range: quantum 2^-9; n == 8 is the smallest normal */
        double n = rint(a * 512.0);
        return sign | (uint8_t)n;
    }
    int ex;
    frexp(a, &ex);              /* a = f * 2^ex, f in [0.5, 1) */
    int e = ex - 1;             /* a in [2^e, 2^(e+1)) */
    double n = rint(ldexp(a, 3 - e));   /* significand in eighths, [8, 16] */
    if (n == 16.0) { e += 1; n = 8.0; }
    return sign | (uint8_t)(((e + 7) << 3) | ((int)n - 8));
}

/* E8M0: unsigned exponent, value 2^(c-127); 255 is NaN. */
float oracle_e8m0_decode(uint8_t c) {
    if (c == 255) return NAN;
    return (float)ldexp(1.0, (int)c - 127);
}

static float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* fp32 -> bf16, round to nearest even (inputs carry no NaN). */
static uint16_t f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

uint16_t oracle_f32_to_bf16(float f) { return f32_to_bf16(f); }

/* ------------------------------------------------------------------ */
/* Stage a1: routing and permutation                                     */
/* ------------------------------------------------------------------ */

/* Router, the step before the expert computation (the AlphaMoE page's
 * five-stage pipeline, "문제점: MoE Expert 계산의 병목", starts from each token's
 * experts and weights).  Reading: a token's k largest logits in descending
 * order, ties to the lower expert index; weights = softmax over those k
 * logits in fp32 with the largest one subtracted (expf), summed in slot
 * order, w_j = e_j / sum. */
void oracle_router_topk(const float* logits, int T, int E, int k, int32_t* ids, float* w) {
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t) {
        const float* l = logits + (size_t)t * E;
        int32_t* id = ids + (size_t)t * k;
        for (int j = 0; j < k; ++j) {
            int best = -1;
            for (int e = 0; e < E; ++e) {
                int taken = 0;
                for (int i = 0; i < j; ++i) taken |= (id[i] == e);
                if (taken) continue;
                if (best < 0 || l[e] > l[best]) best = e;  /* strict: ties keep the lower index */
            }
            id[j] = best;
        }
        float ex[1024];
        float sum = 0.0f;
        const float m = l[id[0]];
        for (int j = 0; j < k; ++j) {
            ex[j] = expf(l[id[j]] - m);
            sum += ex[j];
        }
        for (int j = 0; j < k; ++j) w[(size_t)t * k + j] = ex[j] / sum;
    }
}

/* Group the T*k (token, slot) pairs by expert with a stable counting sort.
 * m_indptr[E+1] is the exclusive prefix of per-expert counts; perm maps a
 * grouped row to its pair id p = t*k + j (ascending p inside each group);
 * inv_perm maps p back to its grouped row.  Pairs whose expert id is outside
 * [0, E) are left out (inv_perm = -1) and counted in the return value. */
int oracle_route_permute(const int32_t* topk_ids, int T, int k, int E,
                         int32_t* m_indptr, int32_t* perm, int32_t* inv_perm) {
    int R = T * k, bad = 0;
    for (int e = 0; e <= E; ++e) m_indptr[e] = 0;
    for (int p = 0; p < R; ++p) {
        int e = topk_ids[p];
        if (e < 0 || e >= E) { ++bad; continue; }
        m_indptr[e + 1] += 1;
    }
    for (int e = 0; e < E; ++e) m_indptr[e + 1] += m_indptr[e];
    int32_t* cursor = (int32_t*)malloc(sizeof(int32_t) * (E > 0 ? E : 1));
    for (int e = 0; e < E; ++e) cursor[e] = m_indptr[e];
    for (int p = 0; p < R; ++p) {
        int e = topk_ids[p];
        if (e < 0 || e >= E) { inv_perm[p] = -1; continue; }
        int row = cursor[e]++;
        perm[row] = p;
        inv_perm[p] = row;
    }
    free(cursor);
    return bad;
}

/* ------------------------------------------------------------------ */
/* Stages a2 / a5: 1x128 block quantisation                              */
/* ------------------------------------------------------------------ */

/* Quantise one block of n fp32 values: scale = amax/448, q = RNE_sat(v/scale). */
static float quant_block(const float* v, int n, uint8_t* q) {
    float amax = 0.0f;
    for (int i = 0; i < n; ++i) {
        float a = fabsf(v[i]);
        if (a > amax) amax = a;
    }
    float s = (amax == 0.0f) ? 1.0f : amax / 448.0f;
    for (int i = 0; i < n; ++i) q[i] = oracle_e4m3_encode(v[i] / s);
    return s;
}

/* Quantise rows of an fp32 matrix [rows, cols] per row per 128 columns.
 * q is [rows, cols]; scale is [rows, cols/128] (row-major). */
void oracle_quant_rows_128(const float* x, int rows, int cols, uint8_t* q, float* scale) {
    int nkb = cols / 128;
    for (int r = 0; r < rows; ++r)
        for (int kb = 0; kb < nkb; ++kb)
            scale[(size_t)r * nkb + kb] =
                quant_block(x + (size_t)r * cols + kb * 128, 128,
                            q + (size_t)r * cols + kb * 128);
}

/* Same for bf16 input rows (activation quantisation, stage a2). */
void oracle_quant_rows_128_bf16(const uint16_t* x, int rows, int cols, uint8_t* q, float* scale) {
    float* row = (float*)malloc(sizeof(float) * cols);
    int nkb = cols / 128;
    for (int r = 0; r < rows; ++r) {
        for (int c = 0; c < cols; ++c) row[c] = bf16_to_f32(x[(size_t)r * cols + c]);
        for (int kb = 0; kb < nkb; ++kb)
            scale[(size_t)r * nkb + kb] =
                quant_block(row + kb * 128, 128, q + (size_t)r * cols + kb * 128);
    }
    free(row);
}

/* ------------------------------------------------------------------ */
/* Stages a3 / a6: grouped block-scaled FP8 GEMM                         */
/* ------------------------------------------------------------------ */

/* One output element: row of A (K codes, K/128 scales) against row n of the
 * expert's B (K codes) with B's scale row for block n/128. */
static float block_scaled_dot(const uint8_t* a, const float* a_s,
                              const uint8_t* b, const float* b_s,
                              int K, const float* dec) {
    float acc = 0.0f;
    for (int kb = 0; kb < K / 128; ++kb) {
        float bsum = 0.0f;
        for (int kk = 0; kk < 128; ++kk) {
            int k = kb * 128 + kk;
            bsum += dec[a[k]] * dec[b[k]];
        }
        float s = a_s[kb] * b_s[kb];
        acc += s * bsum;
    }
    return acc;
}

static void make_decode_table(float* dec) {
    for (int c = 0; c < 256; ++c) dec[c] = oracle_e4m3_decode((uint8_t)c);
}

/* out[r, n] for every grouped row r of expert e (m_indptr rows) and every
 * n < N.  a: [R, K] codes; a_scale: [R, K/128]; b: [E, N, K] codes;
 * b_scale: [E, N/128, K/128]; out: [R, N] fp32. */
void oracle_grouped_gemm(const uint8_t* a, const float* a_scale,
                         const uint8_t* b, const float* b_scale,
                         const int32_t* m_indptr, int R, int N, int K, int E,
                         float* out) {
    float dec[256];
    make_decode_table(dec);
    int nkb = K / 128;
    (void)R;
    int Rg = m_indptr[E];
    #pragma omp parallel for schedule(dynamic, 1)
    for (int r = 0; r < Rg; ++r) {
        int e = 0;
        while (m_indptr[e + 1] <= r) ++e;       /* expert that owns row r */
        for (int n = 0; n < N; ++n)
            out[(size_t)r * N + n] = block_scaled_dot(
                a + (size_t)r * K, a_scale + (size_t)r * nkb,
                b + ((size_t)e * N + n) * K,
                b_scale + ((size_t)e * (N / 128) + n / 128) * nkb, K, dec);
    }
}

/* ------------------------------------------------------------------ */
/* Stage a4: SwiGLU                                                      */
/* ------------------------------------------------------------------ */

static float silu(float z) { return z / (1.0f + expf(-z)); }

/* g: [rows, 2I] with gate = columns [0, I), up = [I, 2I); h: [rows, I]. */
void oracle_swiglu(const float* g, int rows, int I, float* h) {
    for (int r = 0; r < rows; ++r)
        for (int i = 0; i < I; ++i)
            h[(size_t)r * I + i] = silu(g[(size_t)r * 2 * I + i]) * g[(size_t)r * 2 * I + I + i];
}

/* ------------------------------------------------------------------ */
/* The whole layer, grouped form (stages a1..a7)                         */
/* ------------------------------------------------------------------ */

/* x: [T, H] bf16 bits; topk_ids, topk_w: [T, k]; w13: [E, 2I, H] codes with
 * w13_scale [E, 2I/128, H/128]; w2: [E, H, I] codes with w2_scale
 * [E, H/128, I/128]; out: [T, H] bf16 bits.  Optional dumps (NULL to skip):
 * m_indptr [E+1], perm [T*k], h_q [R, I] codes and h_scale [R, I/128] in
 * grouped-row order.  Returns the number of out-of-range expert ids. */
int oracle_moe_fused(const uint16_t* x, const int32_t* topk_ids, const float* topk_w,
                     const uint8_t* w13, const float* w13_scale,
                     const uint8_t* w2, const float* w2_scale,
                     uint16_t* out, int T, int H, int I, int E, int k,
                     int32_t* m_indptr_out, int32_t* perm_out,
                     uint8_t* hq_out, float* hs_out) {
    int R = T * k;
    int32_t* m_indptr = (int32_t*)malloc(sizeof(int32_t) * (E + 1));
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (R > 0 ? R : 1));
    int32_t* inv_perm = (int32_t*)malloc(sizeof(int32_t) * (R > 0 ? R : 1));
    int bad = oracle_route_permute(topk_ids, T, k, E, m_indptr, perm, inv_perm);

    /* a2: quantise each token once, then gather rows in grouped order */
    uint8_t* xq_tok = (uint8_t*)malloc((size_t)T * H + 1);
    float* xs_tok = (float*)malloc(sizeof(float) * ((size_t)T * (H / 128) + 1));
    oracle_quant_rows_128_bf16(x, T, H, xq_tok, xs_tok);
    uint8_t* xq = (uint8_t*)malloc((size_t)R * H + 1);
    float* xs = (float*)malloc(sizeof(float) * ((size_t)R * (H / 128) + 1));
    int Rg = m_indptr[E];
    for (int r = 0; r < Rg; ++r) {
        int t = perm[r] / k;
        memcpy(xq + (size_t)r * H, xq_tok + (size_t)t * H, H);
        memcpy(xs + (size_t)r * (H / 128), xs_tok + (size_t)t * (H / 128), sizeof(float) * (H / 128));
    }

    /* a3: GEMM1 gate/up */
    float* g = (float*)malloc(sizeof(float) * ((size_t)R * 2 * I + 1));
    oracle_grouped_gemm(xq, xs, w13, w13_scale, m_indptr, R, 2 * I, H, E, g);

    /* a4: SwiGLU, a5: requantise the intermediate per row per 128 columns */
    float* h = (float*)malloc(sizeof(float) * ((size_t)R * I + 1));
    oracle_swiglu(g, Rg, I, h);
    uint8_t* hq = (uint8_t*)malloc((size_t)R * I + 1);
    float* hs = (float*)malloc(sizeof(float) * ((size_t)R * (I / 128) + 1));
    oracle_quant_rows_128(h, Rg, I, hq, hs);

    /* a6: GEMM2 down */
    float* y = (float*)malloc(sizeof(float) * ((size_t)R * H + 1));
    oracle_grouped_gemm(hq, hs, w2, w2_scale, m_indptr, R, H, I, E, y);

    /* a7: combine, slots in ascending order */
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < H; ++c) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int row = inv_perm[t * k + j];
                if (row < 0) continue;
                acc += topk_w[t * k + j] * y[(size_t)row * H + c];
            }
            out[(size_t)t * H + c] = f32_to_bf16(acc);
        }

    if (m_indptr_out) memcpy(m_indptr_out, m_indptr, sizeof(int32_t) * (E + 1));
    if (perm_out) memcpy(perm_out, perm, sizeof(int32_t) * Rg);
    if (hq_out) memcpy(hq_out, hq, (size_t)Rg * I);
    if (hs_out) memcpy(hs_out, hs, sizeof(float) * (size_t)Rg * (I / 128));
    free(m_indptr); free(perm); free(inv_perm); free(xq_tok); free(xs_tok);
    free(xq); free(xs); free(g); free(h); free(hq); free(hs); free(y);
    return bad;
}

/* ------------------------------------------------------------------ */
/* The whole layer, per-token form (no grouping)                         */
/* ------------------------------------------------------------------ */

/* Computes the output rows of the listed tokens only, one token and one
 * slot at a time, straight from the definitions: no routing tables, no
 * grouping.  Every token is independent of the others, so this equals the
 * grouped form row for row.  out: [n_tok, H] bf16 bits in list order.
 * hq_out [n_tok*k, I] / hs_out [n_tok*k, I/128] (NULL to skip) receive the
 * requantised intermediate of slot (list index, j). */
void oracle_moe_tokens(const uint16_t* x, const int32_t* topk_ids, const float* topk_w,
                       const uint8_t* w13, const float* w13_scale,
                       const uint8_t* w2, const float* w2_scale,
                       int T, int H, int I, int E, int k,
                       const int32_t* tokens, int n_tok, uint16_t* out,
                       uint8_t* hq_out, float* hs_out) {
    float dec[256];
    make_decode_table(dec);
    (void)T;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_tok; ++it) {
        int t = tokens[it];
        uint8_t* xq = (uint8_t*)malloc(H);
        float* xs = (float*)malloc(sizeof(float) * (H / 128));
        float* g = (float*)malloc(sizeof(float) * 2 * I);
        float* h = (float*)malloc(sizeof(float) * I);
        uint8_t* hq = (uint8_t*)malloc(I);
        float* hs = (float*)malloc(sizeof(float) * (I / 128));
        float* acc = (float*)calloc(H, sizeof(float));
        oracle_quant_rows_128_bf16(x + (size_t)t * H, 1, H, xq, xs);
        for (int j = 0; j < k; ++j) {
            int e = topk_ids[t * k + j];
            if (e < 0 || e >= E) continue;
            for (int n = 0; n < 2 * I; ++n)
                g[n] = block_scaled_dot(xq, xs, w13 + ((size_t)e * 2 * I + n) * H,
                                        w13_scale + ((size_t)e * (2 * I / 128) + n / 128) * (H / 128),
                                        H, dec);
            oracle_swiglu(g, 1, I, h);
            oracle_quant_rows_128(h, 1, I, hq, hs);
            if (hq_out) memcpy(hq_out + ((size_t)it * k + j) * I, hq, I);
            if (hs_out) memcpy(hs_out + ((size_t)it * k + j) * (I / 128), hs, sizeof(float) * (I / 128));
            for (int c = 0; c < H; ++c) {
                float yc = block_scaled_dot(hq, hs, w2 + ((size_t)e * H + c) * I,
                                            w2_scale + ((size_t)e * (H / 128) + c / 128) * (I / 128),
                                            I, dec);
                acc[c] += topk_w[t * k + j] * yc;
            }
        }
        for (int c = 0; c < H; ++c) out[(size_t)it * H + c] = f32_to_bf16(acc[c]);
        free(xq); free(xs); free(g); free(h); free(hq); free(hs); free(acc);
    }
}

/* ------------------------------------------------------------------ */
/* Standalone grouped GEMM with bf16 output (plain or gated)             */
/* ------------------------------------------------------------------ */

/* a_scale_kmajor: [R, K/128].  Plain: out [R, N] = bf16(GEMM).  Gated:
 * out [R, N/2] = bf16(silu(G[:, :N/2]) * G[:, N/2:]). */
void oracle_groupwise_gemm_bf16(const uint8_t* a, const float* a_scale_kmajor,
                                const uint8_t* b, const float* b_scale,
                                const int32_t* m_indptr, int R, int N, int K, int E,
                                int is_gated, uint16_t* out) {
    float* g = (float*)malloc(sizeof(float) * ((size_t)R * N + 1));
    for (size_t i = 0; i < (size_t)R * N; ++i) g[i] = 0.0f;
    oracle_grouped_gemm(a, a_scale_kmajor, b, b_scale, m_indptr, R, N, K, E, g);
    int Rg = m_indptr[E];
    if (!is_gated) {
        for (size_t i = 0; i < (size_t)Rg * N; ++i) out[i] = f32_to_bf16(g[i]);
    } else {
        int I = N / 2;
        float* h = (float*)malloc(sizeof(float) * ((size_t)R * I + 1));
        oracle_swiglu(g, Rg, I, h);
        for (size_t i = 0; i < (size_t)Rg * I; ++i) out[i] = f32_to_bf16(h[i]);
        free(h);
    }
    free(g);
}

/* ------------------------------------------------------------------ */
/* Stage a10: SwiGLU + MXFP8 quantisation                                */
/* ------------------------------------------------------------------ */

/* Smallest integer s with amax <= 448 * 2^s, as an E8M0 code s + 127
 * clamped to [0, 254].  amax == 0 gives code 0. */
uint8_t oracle_e8m0_scale_code(float amax) {
    if (amax == 0.0f) return 0;
    double a = (double)amax;
    int s = (int)ceil(log2(a / 448.0));
    while (a > ldexp(448.0, s)) ++s;            /* exact corrections */
    while (a <= ldexp(448.0, s - 1)) --s;
    int c = s + 127;
    if (c < 0) c = 0;
    if (c > 254) c = 254;
    return (uint8_t)c;
}

/* in: [M, 2K] bf16 bits, gate = columns [0, K), up = [K, 2K).
 * out: [M, K] E4M3 codes; scale: [M, K/32] E8M0 codes (row-major). */
void oracle_swiglu_mxfp8(const uint16_t* in, int M, int K, uint8_t* out, uint8_t* scale) {
    #pragma omp parallel for schedule(static)
    for (int m = 0; m < M; ++m) {
        float v[32];
        for (int b = 0; b < K / 32; ++b) {
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                int c = b * 32 + i;
                float gt = bf16_to_f32(in[(size_t)m * 2 * K + c]);
                float up = bf16_to_f32(in[(size_t)m * 2 * K + K + c]);
                v[i] = silu(gt) * up;
                float a = fabsf(v[i]);
                if (a > amax) amax = a;
            }
            uint8_t code = oracle_e8m0_scale_code(amax);
            float X = oracle_e8m0_decode(code);
            scale[(size_t)m * (K / 32) + b] = code;
            for (int i = 0; i < 32; ++i)
                out[(size_t)m * K + b * 32 + i] = oracle_e4m3_encode(v[i] / X);
        }
    }
}

/* ------------------------------------------------------------------ */
/* MXFP8 variant: one E8M0 scale per 32 consecutive K elements          */
/* ------------------------------------------------------------------ */
/*
 * The Wave page names FP8 and MXFP8 as the two formats of its grouped MoE
 * GEMM (section "들어가며"; "mxfp8 grouped MoE" timings in "왜 이게 좋은가?").
 * MXFP8 scales every 32 consecutive elements along K with a power of two
 * (E8M0), on both operands; the scale rule is the one above (the Cake-act
 * page's SwiGLU + MXFP8 kernel).  Products of two E4M3 values and their sum
 * over a 32-element block are exact in double, and so is the power-of-two
 * scaling; the blocks are accumulated in double and the result rounded to
 * fp32 once.  The tensor core accumulates in fp32, so the two agree to a
 * tolerance, not bit for bit.
 */

/* x: [rows, cols] bf16 bits, cols a multiple of 32.  q: [rows, cols] E4M3
 * codes; sf: [rows, cols/32] E8M0 codes (row-major). */
void oracle_quant_rows_mx_bf16(const uint16_t* x, int rows, int cols, uint8_t* q, uint8_t* sf) {
    #pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        for (int b = 0; b < cols / 32; ++b) {
            float v[32];
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                v[i] = bf16_to_f32(x[(size_t)r * cols + b * 32 + i]);
                float a = fabsf(v[i]);
                if (a > amax) amax = a;
            }
            uint8_t code = oracle_e8m0_scale_code(amax);
            float X = oracle_e8m0_decode(code);
            sf[(size_t)r * (cols / 32) + b] = code;
            for (int i = 0; i < 32; ++i)
                q[(size_t)r * cols + b * 32 + i] = oracle_e4m3_encode(v[i] / X);
        }
    }
}

/* fp32 rows -> MXFP8 (same rule as oracle_quant_rows_mx_bf16). */
static void quant_rows_mx_f32(const float* x, int rows, int cols, uint8_t* q, uint8_t* sf) {
    #pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        for (int b = 0; b < cols / 32; ++b) {
            const float* v = x + (size_t)r * cols + b * 32;
            float amax = 0.0f;
            for (int i = 0; i < 32; ++i) {
                float a = fabsf(v[i]);
                if (a > amax) amax = a;
            }
            uint8_t code = oracle_e8m0_scale_code(amax);
            float X = oracle_e8m0_decode(code);
            sf[(size_t)r * (cols / 32) + b] = code;
            for (int i = 0; i < 32; ++i)
                q[(size_t)r * cols + b * 32 + i] = oracle_e4m3_encode(v[i] / X);
        }
    }
}

/* Grouped MXFP8 GEMM in the m_indptr layout.  a: [R, K] codes, a_sf [R, K/32];
 * b: [E, N, K] codes, b_sf [E, N, K/32]; rows [m_indptr[e], m_indptr[e+1])
 * use expert e.  out: [R, N] fp32 (rows outside every group untouched). */
void oracle_mx_grouped_gemm(const uint8_t* a, const uint8_t* a_sf, const uint8_t* b,
                            const uint8_t* b_sf, const int32_t* m_indptr, int R, int N, int K,
                            int E, float* out) {
    float dec[256];
    make_decode_table(dec);
    const int nb = K / 32;
    (void)R;
    for (int e = 0; e < E; ++e) {
        #pragma omp parallel for schedule(static)
        for (int r = m_indptr[e]; r < m_indptr[e + 1]; ++r) {
            const uint8_t* ar = a + (size_t)r * K;
            for (int n = 0; n < N; ++n) {
                const size_t wrow = (size_t)e * N + n;
                const uint8_t* br = b + wrow * K;
                double acc = 0.0;
                for (int blk = 0; blk < nb; ++blk) {
                    double s = 0.0;
                    for (int i = 0; i < 32; ++i)
                        s += (double)dec[ar[blk * 32 + i]] * (double)dec[br[blk * 32 + i]];
                    const int ex = (int)a_sf[(size_t)r * nb + blk] + (int)b_sf[wrow * nb + blk] - 254;
                    acc += ldexp(s, ex);
                }
                out[(size_t)r * N + n] = (float)acc;
            }
        }
    }
}

/* bf16 output of the MXFP8 GEMM: plain out [R, N], or gated out [R, N/2] =
 * bf16(silu(G[:, :N/2]) * G[:, N/2:]) with G rounded to fp32 first. */
void oracle_mx_gemm_bf16(const uint8_t* a, const uint8_t* a_sf, const uint8_t* b,
                         const uint8_t* b_sf, const int32_t* m_indptr, int R, int N, int K, int E,
                         int is_gated, uint16_t* out) {
    float* g = (float*)malloc(sizeof(float) * ((size_t)R * N + 1));
    for (size_t i = 0; i < (size_t)R * N; ++i) g[i] = 0.0f;
    oracle_mx_grouped_gemm(a, a_sf, b, b_sf, m_indptr, R, N, K, E, g);
    int Rg = m_indptr[E];
    if (!is_gated) {
        for (size_t i = 0; i < (size_t)Rg * N; ++i) out[i] = f32_to_bf16(g[i]);
    } else {
        int I = N / 2;
        float* h = (float*)malloc(sizeof(float) * ((size_t)R * I + 1));
        oracle_swiglu(g, Rg, I, h);
        for (size_t i = 0; i < (size_t)Rg * I; ++i) out[i] = f32_to_bf16(h[i]);
        free(h);
    }
    free(g);
}

/* The fused layer in the MXFP8 variant: the five stages of the AlphaMoE
 * page's pipeline ("문제점: MoE Expert 계산의 병목", stages 1-5) with every FP8
 * operand in MXFP8 (E8M0 per 32 K elements): activations quantised per
 * token per 32 columns and gathered into grouped rows, GEMM1 gate/up, SwiGLU
 * in fp32, requantisation of the intermediate to MXFP8 per row per 32
 * columns (the Cake-act page's SwiGLU + MXFP8 rule), GEMM2 down, combine in
 * fp32 (ascending slot) and bf16.  Weight scales row-major:
 * w13_sf [E, 2I, H/32], w2_sf [E, H, I/32].  Optional dumps: m_indptr [E+1],
 * perm [R], hq [R, I] codes, hsf [R, I/32]. */
int oracle_moe_mx_fused(const uint16_t* x, const int32_t* topk_ids, const float* topk_w,
                        const uint8_t* w13, const uint8_t* w13_sf,
                        const uint8_t* w2, const uint8_t* w2_sf,
                        uint16_t* out, int T, int H, int I, int E, int k,
                        int32_t* m_indptr_out, int32_t* perm_out,
                        uint8_t* hq_out, uint8_t* hsf_out) {
    int R = T * k;
    int32_t* m_indptr = (int32_t*)malloc(sizeof(int32_t) * (E + 1));
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (R > 0 ? R : 1));
    int32_t* inv_perm = (int32_t*)malloc(sizeof(int32_t) * (R > 0 ? R : 1));
    int bad = oracle_route_permute(topk_ids, T, k, E, m_indptr, perm, inv_perm);
    int Rg = m_indptr[E];

    uint8_t* xq_tok = (uint8_t*)malloc((size_t)T * H + 1);
    uint8_t* xsf_tok = (uint8_t*)malloc((size_t)T * (H / 32) + 1);
    oracle_quant_rows_mx_bf16(x, T, H, xq_tok, xsf_tok);
    uint8_t* xq = (uint8_t*)malloc((size_t)R * H + 1);
    uint8_t* xsf = (uint8_t*)malloc((size_t)R * (H / 32) + 1);
    for (int r = 0; r < Rg; ++r) {
        int t = perm[r] / k;
        memcpy(xq + (size_t)r * H, xq_tok + (size_t)t * H, H);
        memcpy(xsf + (size_t)r * (H / 32), xsf_tok + (size_t)t * (H / 32), H / 32);
    }
    float* g = (float*)malloc(sizeof(float) * ((size_t)R * 2 * I + 1));
    oracle_mx_grouped_gemm(xq, xsf, w13, w13_sf, m_indptr, R, 2 * I, H, E, g);
    float* h = (float*)malloc(sizeof(float) * ((size_t)R * I + 1));
    oracle_swiglu(g, Rg, I, h);
    uint8_t* hq = (uint8_t*)malloc((size_t)R * I + 1);
    uint8_t* hsf = (uint8_t*)malloc((size_t)R * (I / 32) + 1);
    quant_rows_mx_f32(h, Rg, I, hq, hsf);
    float* y = (float*)malloc(sizeof(float) * ((size_t)R * H + 1));
    oracle_mx_grouped_gemm(hq, hsf, w2, w2_sf, m_indptr, R, H, I, E, y);
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < H; ++c) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int row = inv_perm[t * k + j];
                if (row < 0) continue;
                acc += topk_w[t * k + j] * y[(size_t)row * H + c];
            }
            out[(size_t)t * H + c] = f32_to_bf16(acc);
        }
    if (m_indptr_out) memcpy(m_indptr_out, m_indptr, sizeof(int32_t) * (E + 1));
    if (perm_out) memcpy(perm_out, perm, sizeof(int32_t) * Rg);
    if (hq_out) memcpy(hq_out, hq, (size_t)Rg * I);
    if (hsf_out) memcpy(hsf_out, hsf, (size_t)Rg * (I / 32));
    free(m_indptr); free(perm); free(inv_perm); free(xq_tok); free(xsf_tok);
    free(xq); free(xsf); free(g); free(h); free(hq); free(hsf); free(y);
    return bad;
}

/* One 32-wide-block-scaled dot product of length K, as in
 * oracle_mx_grouped_gemm (block sums and power-of-two scaling exact in
 * double, blocks accumulated in double). */
static double mx_dot(const uint8_t* a, const uint8_t* a_sf, const uint8_t* b, const uint8_t* b_sf,
                     int K, const float* dec) {
    double acc = 0.0;
    for (int blk = 0; blk < K / 32; ++blk) {
        double s = 0.0;
        for (int i = 0; i < 32; ++i)
            s += (double)dec[a[blk * 32 + i]] * (double)dec[b[blk * 32 + i]];
        acc += ldexp(s, (int)a_sf[blk] + (int)b_sf[blk] - 254);
    }
    return acc;
}

/* The MXFP8 layer for selected tokens only, one token at a time (no
 * grouping): same arithmetic as oracle_moe_mx_fused for each of their rows.
 * w13_sf [E, 2I, H/32], w2_sf [E, H, I/32] row-major.  out [n_tok, H] bf16;
 * optional hq [n_tok*k, I], hsf [n_tok*k, I/32] (slot order). */
void oracle_moe_mx_tokens(const uint16_t* x, const int32_t* topk_ids, const float* topk_w,
                          const uint8_t* w13, const uint8_t* w13_sf,
                          const uint8_t* w2, const uint8_t* w2_sf,
                          int T, int H, int I, int E, int k,
                          const int32_t* tokens, int n_tok, uint16_t* out,
                          uint8_t* hq_out, uint8_t* hsf_out) {
    float dec[256];
    make_decode_table(dec);
    (void)T;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_tok; ++it) {
        int t = tokens[it];
        uint8_t* xq = (uint8_t*)malloc(H);
        uint8_t* xsf = (uint8_t*)malloc(H / 32);
        float* g = (float*)malloc(sizeof(float) * 2 * I);
        float* h = (float*)malloc(sizeof(float) * I);
        uint8_t* hq = (uint8_t*)malloc(I);
        uint8_t* hsf = (uint8_t*)malloc(I / 32);
        float* acc = (float*)calloc(H, sizeof(float));
        oracle_quant_rows_mx_bf16(x + (size_t)t * H, 1, H, xq, xsf);
        for (int j = 0; j < k; ++j) {
            int e = topk_ids[t * k + j];
            if (e < 0 || e >= E) continue;
            for (int n = 0; n < 2 * I; ++n) {
                const size_t wr = (size_t)e * 2 * I + n;
                g[n] = (float)mx_dot(xq, xsf, w13 + wr * H, w13_sf + wr * (H / 32), H, dec);
            }
            oracle_swiglu(g, 1, I, h);
            quant_rows_mx_f32(h, 1, I, hq, hsf);
            if (hq_out) memcpy(hq_out + ((size_t)it * k + j) * I, hq, I);
            if (hsf_out) memcpy(hsf_out + ((size_t)it * k + j) * (I / 32), hsf, I / 32);
            for (int c = 0; c < H; ++c) {
                const size_t wr = (size_t)e * H + c;
                float yc = (float)mx_dot(hq, hsf, w2 + wr * I, w2_sf + wr * (I / 32), I, dec);
                acc[c] += topk_w[t * k + j] * yc;
            }
        }
        for (int c = 0; c < H; ++c) out[(size_t)it * H + c] = f32_to_bf16(acc[c]);
        free(xq); free(xsf); free(g); free(h); free(hq); free(hsf); free(acc);
    }
}

/* ------------------------------------------------------------------ */
/* NVFP4 variant: FP4 E2M1 values, one E4M3 scale per 16 elements and   */
/* one fp32 global scale per tensor (per expert for weights)            */
/* ------------------------------------------------------------------ */
/*
 * The cuTile page ("FlashInfer에 cuTile 기반 Fused MoE 백엔드 도입", section
 * "2. cuTile NVFP4 양자화 지원") quantises the experts to NVFP4 (W4A4) with
 * fp4_quantize(weight, global_scale=<per expert>, sf_vec_size=16); it gives
 * no formulas.  Reading taken here (the format's published definition):
 *  - E2M1: sign, 2 exponent bits (bias 1), 1 mantissa bit; magnitudes
 *    0, 0.5, 1, 1.5, 2, 3, 4, 6 (0.5 is the subnormal); no inf/NaN.
 *  - the global scale g multiplies the data into range (g = 448*6/amax of
 *    the tensor is the usual choice, passed in);
 *  - per 16 consecutive elements: scale code c = E4M3_RNE_sat(amax_block * g / 6)
 *    (an all-zero block gets c = 0);
 *  - codes q = E2M1_RNE_sat(x * g / dec(c)) (q = 0 where dec(c) = 0);
 *  - dequantised value = dec_e2m1(q) * dec_e4m3(c) / g.
 */
static const float kE2M1[8] = {0.0f, 0.5f, 1.0f, 1.5f, 2.0f, 3.0f, 4.0f, 6.0f};

float oracle_e2m1_decode(uint8_t c) {
    float v = kE2M1[c & 7];
    return (c & 8) ? -v : v;
}

/* Round to the nearest E2M1 value, ties to the even code, saturating at 6. */
uint8_t oracle_e2m1_encode(float v) {
    uint8_t sign = (v < 0.0f || (v == 0.0f && signbit(v))) ? 8 : 0;
    float a = fabsf(v);
    if (!(a == a)) return sign;  /* NaN: not produced by finite inputs */
    uint8_t best = 0;
    for (uint8_t c = 1; c < 8; ++c) {
        float d = fabsf(a - kE2M1[c]), db = fabsf(a - kE2M1[best]);
        if (d < db || (d == db && (c & 1) == 0)) best = c;
    }
    return (uint8_t)(sign | best);
}

/* x [rows, cols] fp32, cols a multiple of 16; g the global scale.
 * q [rows, cols] E2M1 codes (one per byte, low 4 bits); sf [rows, cols/16]
 * E4M3 codes. */
void oracle_quant_rows_nvfp4(const float* x, int rows, int cols, float g, uint8_t* q, uint8_t* sf) {
    #pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        for (int b = 0; b < cols / 16; ++b) {
            const float* v = x + (size_t)r * cols + b * 16;
            float amax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(v[i]);
                if (a > amax) amax = a;
            }
            uint8_t c = oracle_e4m3_encode(amax * g / 6.0f);
            float s = oracle_e4m3_decode(c);
            sf[(size_t)r * (cols / 16) + b] = c;
            for (int i = 0; i < 16; ++i)
                q[(size_t)r * cols + b * 16 + i] = s > 0.0f ? oracle_e2m1_encode(v[i] * g / s) : 0;
        }
    }
}

/* Grouped NVFP4 GEMM in the m_indptr layout: per 16-wide K block,
 * dec(sa) dec(sb) / (ga gb_e) times the block dot of the E2M1 values, in
 * double, rounded to fp32 once.  a [R, K] codes, a_sf [R, K/16], ga;
 * b [E, N, K] codes, b_sf [E, N, K/16], gb [E]. */
void oracle_nvfp4_grouped_gemm(const uint8_t* a, const uint8_t* a_sf, float ga, const uint8_t* b,
                               const uint8_t* b_sf, const float* gb, const int32_t* m_indptr,
                               int R, int N, int K, int E, float* out) {
    float dec[256];
    make_decode_table(dec);
    const int nb = K / 16;
    (void)R;
    for (int e = 0; e < E; ++e) {
        #pragma omp parallel for schedule(static)
        for (int r = m_indptr[e]; r < m_indptr[e + 1]; ++r) {
            for (int n = 0; n < N; ++n) {
                const size_t wrow = (size_t)e * N + n;
                double acc = 0.0;
                for (int blk = 0; blk < nb; ++blk) {
                    double s = 0.0;
                    for (int i = 0; i < 16; ++i)
                        s += (double)oracle_e2m1_decode(a[(size_t)r * K + blk * 16 + i]) *
                             (double)oracle_e2m1_decode(b[wrow * K + blk * 16 + i]);
                    acc += s * (double)dec[a_sf[(size_t)r * nb + blk]] *
                           (double)dec[b_sf[wrow * nb + blk]];
                }
                out[(size_t)r * N + n] = (float)(acc / ((double)ga * (double)gb[e]));
            }
        }
    }
}

/* bf16 output of the NVFP4 GEMM, as oracle_mx_gemm_bf16: plain out [R, N],
 * or gated out [R, N/2] = bf16(silu(G[:, :N/2]) * G[:, N/2:]) with G (global
 * scales applied) rounded to fp32 first. */
void oracle_nvfp4_gemm_bf16(const uint8_t* a, const uint8_t* a_sf, float ga, const uint8_t* b,
                            const uint8_t* b_sf, const float* gb, const int32_t* m_indptr,
                            int R, int N, int K, int E, int is_gated, uint16_t* out) {
    float* g = (float*)malloc(sizeof(float) * ((size_t)R * N + 1));
    for (size_t i = 0; i < (size_t)R * N; ++i) g[i] = 0.0f;
    oracle_nvfp4_grouped_gemm(a, a_sf, ga, b, b_sf, gb, m_indptr, R, N, K, E, g);
    int Rg = m_indptr[E];
    if (!is_gated) {
        for (size_t i = 0; i < (size_t)Rg * N; ++i) out[i] = f32_to_bf16(g[i]);
    } else {
        int I = N / 2;
        float* h = (float*)malloc(sizeof(float) * ((size_t)R * I + 1));
        oracle_swiglu(g, Rg, I, h);
        for (size_t i = 0; i < (size_t)Rg * I; ++i) out[i] = f32_to_bf16(h[i]);
        free(h);
    }
    free(g);
}

/* x [rows, cols] bf16 bits -> NVFP4 codes and scales with global scale g
 * (oracle_quant_rows_nvfp4 on the exact fp32 values of x). */
static void quant_rows_nvfp4_bf16(const uint16_t* x, int rows, int cols, float g, uint8_t* q,
                                  uint8_t* sf) {
    float* xf = (float*)malloc(sizeof(float) * ((size_t)rows * cols + 1));
    for (size_t i = 0; i < (size_t)rows * cols; ++i) xf[i] = bf16_to_f32(x[i]);
    oracle_quant_rows_nvfp4(xf, rows, cols, g, q, sf);
    free(xf);
}

/* The fused layer in the NVFP4 (W4A4) variant: the five stages of the
 * AlphaMoE page's pipeline ("문제점: MoE Expert 계산의 병목", stages 1-5) with
 * every operand in NVFP4 as the cuTile page quantises it ("2. cuTile NVFP4
 * 양자화 지원"): x quantised per token per 16 columns with the global scale
 * a1_g and gathered into grouped rows, GEMM1 gate/up (weights w13 with
 * per-expert global scales w13_g), SwiGLU in fp32, the intermediate
 * requantised per row per 16 columns with the global scale a2_g, GEMM2 down
 * (w2, w2_g), combine in fp32 (ascending slot) and bf16.  Codes one per byte;
 * scales row-major: w13_sf [E, 2I, H/16], w2_sf [E, H, I/16].  Optional dumps:
 * m_indptr [E+1], perm [R], hq [R, I] codes, hsf [R, I/16]. */
int oracle_moe_nvfp4_fused(const uint16_t* x, const int32_t* topk_ids, const float* topk_w,
                           const uint8_t* w13, const uint8_t* w13_sf, const float* w13_g,
                           const uint8_t* w2, const uint8_t* w2_sf, const float* w2_g,
                           float a1_g, float a2_g, uint16_t* out, int T, int H, int I, int E,
                           int k, int32_t* m_indptr_out, int32_t* perm_out, uint8_t* hq_out,
                           uint8_t* hsf_out) {
    int R = T * k;
    int32_t* m_indptr = (int32_t*)malloc(sizeof(int32_t) * (E + 1));
    int32_t* perm = (int32_t*)malloc(sizeof(int32_t) * (R > 0 ? R : 1));
    int32_t* inv_perm = (int32_t*)malloc(sizeof(int32_t) * (R > 0 ? R : 1));
    int bad = oracle_route_permute(topk_ids, T, k, E, m_indptr, perm, inv_perm);
    int Rg = m_indptr[E];

    uint8_t* xq_tok = (uint8_t*)malloc((size_t)T * H + 1);
    uint8_t* xsf_tok = (uint8_t*)malloc((size_t)T * (H / 16) + 1);
    quant_rows_nvfp4_bf16(x, T, H, a1_g, xq_tok, xsf_tok);
    uint8_t* xq = (uint8_t*)malloc((size_t)R * H + 1);
    uint8_t* xsf = (uint8_t*)malloc((size_t)R * (H / 16) + 1);
    for (int r = 0; r < Rg; ++r) {
        int t = perm[r] / k;
        memcpy(xq + (size_t)r * H, xq_tok + (size_t)t * H, H);
        memcpy(xsf + (size_t)r * (H / 16), xsf_tok + (size_t)t * (H / 16), H / 16);
    }
    float* g = (float*)malloc(sizeof(float) * ((size_t)R * 2 * I + 1));
    oracle_nvfp4_grouped_gemm(xq, xsf, a1_g, w13, w13_sf, w13_g, m_indptr, R, 2 * I, H, E, g);
    float* h = (float*)malloc(sizeof(float) * ((size_t)R * I + 1));
    oracle_swiglu(g, Rg, I, h);
    uint8_t* hq = (uint8_t*)malloc((size_t)R * I + 1);
    uint8_t* hsf = (uint8_t*)malloc((size_t)R * (I / 16) + 1);
    oracle_quant_rows_nvfp4(h, Rg, I, a2_g, hq, hsf);
    float* y = (float*)malloc(sizeof(float) * ((size_t)R * H + 1));
    oracle_nvfp4_grouped_gemm(hq, hsf, a2_g, w2, w2_sf, w2_g, m_indptr, R, H, I, E, y);
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < H; ++c) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int row = inv_perm[t * k + j];
                if (row < 0) continue;
                acc += topk_w[t * k + j] * y[(size_t)row * H + c];
            }
            out[(size_t)t * H + c] = f32_to_bf16(acc);
        }
    if (m_indptr_out) memcpy(m_indptr_out, m_indptr, sizeof(int32_t) * (E + 1));
    if (perm_out) memcpy(perm_out, perm, sizeof(int32_t) * Rg);
    if (hq_out) memcpy(hq_out, hq, (size_t)Rg * I);
    if (hsf_out) memcpy(hsf_out, hsf, (size_t)Rg * (I / 16));
    free(m_indptr); free(perm); free(inv_perm); free(xq_tok); free(xsf_tok);
    free(xq); free(xsf); free(g); free(h); free(hq); free(hsf); free(y);
    return bad;
}

/* One NVFP4 dot product of length K, as in oracle_nvfp4_grouped_gemm: block
 * sums and scale products in double, blocks accumulated in double, then
 * divided by the product of the global scales and rounded to fp32. */
static float nvfp4_dot(const uint8_t* a, const uint8_t* a_sf, float ga, const uint8_t* b,
                       const uint8_t* b_sf, float gb, int K, const float* dec) {
    double acc = 0.0;
    for (int blk = 0; blk < K / 16; ++blk) {
        double s = 0.0;
        for (int i = 0; i < 16; ++i)
            s += (double)oracle_e2m1_decode(a[blk * 16 + i]) * (double)oracle_e2m1_decode(b[blk * 16 + i]);
        acc += s * (double)dec[a_sf[blk]] * (double)dec[b_sf[blk]];
    }
    return (float)(acc / ((double)ga * (double)gb));
}

/* The NVFP4 layer for selected tokens only, one token at a time (no
 * grouping): same arithmetic as oracle_moe_nvfp4_fused for each of their
 * rows.  out [n_tok, H] bf16; optional hq [n_tok*k, I], hsf [n_tok*k, I/16]
 * (slot order). */
void oracle_moe_nvfp4_tokens(const uint16_t* x, const int32_t* topk_ids, const float* topk_w,
                             const uint8_t* w13, const uint8_t* w13_sf, const float* w13_g,
                             const uint8_t* w2, const uint8_t* w2_sf, const float* w2_g,
                             float a1_g, float a2_g, int T, int H, int I, int E, int k,
                             const int32_t* tokens, int n_tok, uint16_t* out, uint8_t* hq_out,
                             uint8_t* hsf_out) {
    float dec[256];
    make_decode_table(dec);
    (void)T;
    #pragma omp parallel for schedule(dynamic, 1)
    for (int it = 0; it < n_tok; ++it) {
        int t = tokens[it];
        uint8_t* xq = (uint8_t*)malloc(H);
        uint8_t* xsf = (uint8_t*)malloc(H / 16);
        float* g = (float*)malloc(sizeof(float) * 2 * I);
        float* h = (float*)malloc(sizeof(float) * I);
        uint8_t* hq = (uint8_t*)malloc(I);
        uint8_t* hsf = (uint8_t*)malloc(I / 16);
        float* acc = (float*)calloc(H, sizeof(float));
        quant_rows_nvfp4_bf16(x + (size_t)t * H, 1, H, a1_g, xq, xsf);
        for (int j = 0; j < k; ++j) {
            int e = topk_ids[t * k + j];
            if (e < 0 || e >= E) continue;
            for (int n = 0; n < 2 * I; ++n) {
                const size_t wr = (size_t)e * 2 * I + n;
                g[n] = nvfp4_dot(xq, xsf, a1_g, w13 + wr * H, w13_sf + wr * (H / 16), w13_g[e], H, dec);
            }
            oracle_swiglu(g, 1, I, h);
            oracle_quant_rows_nvfp4(h, 1, I, a2_g, hq, hsf);
            if (hq_out) memcpy(hq_out + ((size_t)it * k + j) * I, hq, I);
            if (hsf_out) memcpy(hsf_out + ((size_t)it * k + j) * (I / 16), hsf, I / 16);
            for (int c = 0; c < H; ++c) {
                const size_t wr = (size_t)e * H + c;
                float yc = nvfp4_dot(hq, hsf, a2_g, w2 + wr * I, w2_sf + wr * (I / 16), w2_g[e], I, dec);
                acc[c] += topk_w[t * k + j] * yc;
            }
        }
        for (int c = 0; c < H; ++c) out[(size_t)it * H + c] = f32_to_bf16(acc[c]);
        free(xq); free(xsf); free(g); free(h); free(hq); free(hsf); free(acc);
    }
}

/* Threads an OpenMP parallel region would use (0 when built without it). */
int oracle_num_threads(void) {
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------ */
/* Stage 5 on its own: the top-k weighted combine                        */
/* ------------------------------------------------------------------ */

/* The AlphaMoE page's last stage ("문제점: MoE Expert 계산의 병목", stage 5):
 * out[t, c] = bf16( sum_j topk_w[t, j] * y[inv_perm[t*k + j], c] ), the
 * products and the sum in fp32, slots in ascending j, pairs with
 * inv_perm < 0 (dropped ids) skipped.  y [rows, H] fp32 in grouped-row order;
 * out [T, H] bf16 bits.  The same loop ends oracle_moe_fused; here it takes a
 * y from elsewhere (for example GEMM2 recomputed on another intermediate). */
void oracle_combine(const float* y, const int32_t* inv_perm, const float* topk_w, int T, int k,
                    int H, uint16_t* out) {
    #pragma omp parallel for schedule(static)
    for (int t = 0; t < T; ++t)
        for (int c = 0; c < H; ++c) {
            float acc = 0.0f;
            for (int j = 0; j < k; ++j) {
                int row = inv_perm[t * k + j];
                if (row < 0) continue;
                acc += topk_w[t * k + j] * y[(size_t)row * H + c];
            }
            out[(size_t)t * H + c] = f32_to_bf16(acc);
        }
}
