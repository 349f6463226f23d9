/*
 * CPU oracle for the MosaicQuant / ZipperEngine hot path.
 *
 * TEST INFRASTRUCTURE ONLY. Only the test suite, the package smoke check and the
 * benchmark's CPU-baseline leg may load this library. The CUDA product path never
 * calls it and shares no code, header or table with it.
 *
 * Plain, slow, obviously correct definitions, in the order the method states them:
 *
 *  - MosaicQuant decomposes the (outlier-migrated) weight matrix into a dense 4-bit
 *    base Q(W) plus a 4-bit residual R that compensates the base's quantization
 *    error, W ~ Q(W) + R (MosaicQuant technical summary, "Methodology",
 *    section 1 "Inlier-outlier disaggregation"; arXiv abstract of 2606.15652).
 *  - The residual is kept only on the top-K weight blocks ranked by a
 *    Hessian-guided Delta-score: the marginal output-distortion reduction of a block,
 *    residual error weighted by the diagonal-Hessian activation sensitivity of the
 *    input channels (summary, "Methodology", section 2 "Block-wise residual
 *    allocation").
 *  - ZipperEngine computes dense base and sparse residual blocks into one output
 *    (summary, "Methodology", section 3 "ZipperEngine").
 *
 * The pages do not fix the 4-bit format, the block size or the Delta formula; this
 * oracle uses NVFP4 (E2M1 values, one E4M3 scale per 16 consecutive K elements, an
 * fp32 tensor scale), 64x64 (N x K) blocks and
 *     Delta_b = sum_{(n,k) in b} H_k * [ e_nk^2 - e'_nk^2 ],
 *     e = W - deq Q(W),  e' = e - deq R,  H_k = mean_t x_tk^2.
 * NVFP4 is the format the ARCQuant summary names as native to Blackwell, with
 * 16-element blocks and an E2M1 mantissa ("Problem" section of that page).
 *
 * Arithmetic: fp32 IEEE operations exactly as written (compile with
 * -ffp-contract=off, no fast-math, no fused multiply-add), fp64 where stated.
 * Rounding is RNE throughout.
 *
 * Parity pins (tests/test_oracle_*.py): grid round trips and tie tables against a
 * brute-force nearest-value search, torch's float8 conversion, closed-form error
 * bounds, the lossless special case (GEMM == plain matmul of the inputs),
 * budget 0 == dense base, linearity, Delta >= 0 and the exact distortion identity
 * E(S) = E(empty) - sum_{b in S} Delta_b, brute-force top-K over all subsets, pack
 * round trip and an independent unswizzle of the tiled scale layout.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------------ */
/* Number formats                                                                  */
/* ------------------------------------------------------------------------------ */

/* E2M1 value of a 4-bit code: bit 3 sign, bits 2..1 exponent (bias 1), bit 0
 * mantissa. Exponent 0 is subnormal: m * 0.5. Grid {0,0.5,1,1.5,2,3,4,6}. */
double orc_e2m1_value(uint8_t code) {
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    double v = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -v : v;
}

/* E2M1 encode: round to nearest, ties to the even code, saturate at 6, keep the
 * sign (so -0.1 -> 0x8). Thresholds are the midpoints of the grid. */
uint8_t orc_e2m1_encode(float v) {
    uint8_t s = signbit(v) ? 8 : 0;
    float a = fabsf(v);
    uint8_t m;
    if (a <= 0.25f) m = 0;       /* tie 0.25 -> 0   (code 0 even) */
    else if (a < 0.75f) m = 1;   /* 0.5 */
    else if (a <= 1.25f) m = 2;  /* tie 0.75 -> 1, tie 1.25 -> 1 */
    else if (a < 1.75f) m = 3;   /* 1.5 */
    else if (a <= 2.5f) m = 4;   /* tie 1.75 -> 2, tie 2.5 -> 2 */
    else if (a < 3.5f) m = 5;    /* 3 */
    else if (a <= 5.0f) m = 6;   /* tie 3.5 -> 4, tie 5 -> 4 */
    else m = 7;                  /* 6, satfinite */
    return (uint8_t)(s | m);
}

/* E4M3 (the "fn" variant: no infinities, 0x7F/0xFF are NaN) value of a byte:
 * bias 7, exponent 0 subnormal (m * 2^-9), max 448. */
double orc_e4m3_value(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 15, m = code & 7;
    double v = (e == 0) ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
    return s ? -v : v;
}

/* E4M3 encode, round to nearest even, saturating to +-448 (never NaN). */
uint8_t orc_e4m3_encode(float v) {
    uint8_t s = signbit(v) ? 0x80 : 0;
    double a = fabs((double)v);
    if (a == 0.0) return s;
    int e;
    frexp(a, &e);             /* a = f * 2^e, f in [0.5, 1): binade exponent e - 1 */
    int E = e - 1;
    if (E < -6) E = -6;       /* below the normal range the quantum stays 2^-9 */
    double q = ldexp(1.0, E - 3);
    double r = rint(a / q) * q; /* a / q is exact (power of two); rint is RNE */
    if (r > 448.0) r = 448.0;
    if (r == 0.0) return s;
    frexp(r, &e);
    E = e - 1;
    if (E < -6) return (uint8_t)(s | (int)(r * 512.0)); /* subnormal: m * 2^-9 */
    int m = (int)(ldexp(r, -E) * 8.0) - 8;
    return (uint8_t)(s | ((E + 7) << 3) | m);
}

static inline float bf16_to_f32(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, 4);
    return f;
}

/* ------------------------------------------------------------------------------ */
/* NVFP4 quantization                                                              */
/* ------------------------------------------------------------------------------ */

/* Tensor scale g = amax / (6 * 448), so the largest group scale lands on the E4M3
 * maximum; g = 1 for an all-zero tensor. */
float orc_global_scale_f32(const float* a, int64_t n) {
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) amax = fmaxf(amax, fabsf(a[i]));
    return amax == 0.0f ? 1.0f : amax / 2688.0f;
}

/* One 16-element group with tensor scale g, fp32 ops in this order:
 *   amax = max|a_i|;  g6 = 6*g;  s = amax / g6;  sf = E4M3(s);  d = dec(sf) * g;
 *   r = 1 / d;  code_i = E2M1(a_i * r) if d > 0, else a signed zero;
 *   deq_i = val(code_i) * d.
 * The scaled value is a_i times the group's reciprocal (one division per group, the
 * usual form of a block-scaled quantizer), not a per-element division.
 * Writes 16 codes (one per byte, unpacked), the scale byte and the dequantized values. */
static void nvfp4_group(const float* a, float g, uint8_t* codes, uint8_t* sf, float* deq) {
    float amax = 0.0f;
    for (int i = 0; i < 16; ++i) amax = fmaxf(amax, fabsf(a[i]));
    float g6 = 6.0f * g;
    float s_raw = amax / g6;
    uint8_t sfc = orc_e4m3_encode(s_raw);
    float sd = (float)orc_e4m3_value(sfc);
    float d = sd * g;
    float r = (d > 0.0f) ? 1.0f / d : 0.0f;
    for (int i = 0; i < 16; ++i) {
        uint8_t c = (d > 0.0f) ? orc_e2m1_encode(a[i] * r) : (uint8_t)(signbit(a[i]) ? 8 : 0);
        codes[i] = c;
        deq[i] = (float)orc_e2m1_value(c) * d;
    }
    *sf = sfc;
}

/* Pack 16 unpacked codes of group `grp` into a row of packed bytes: element 2j in
 * the low nibble of byte j, element 2j+1 in the high nibble. */
static void pack_group(const uint8_t* c16, uint8_t* row_codes, int64_t grp) {
    for (int j = 0; j < 8; ++j)
        row_codes[grp * 8 + j] = (uint8_t)((c16[2 * j] & 15) | ((c16[2 * j + 1] & 15) << 4));
}

/* Quantize rows x cols fp32 values with per-row scales g[r * g_stride]
 * (g_stride = 0: one tensor scale). Outputs packed codes [rows][cols/2], scales
 * [rows][cols/16] and, if deq != NULL, dequantized fp32 values [rows][cols]. */
void orc_nvfp4_quantize(const float* a, int rows, int cols, const float* g, int g_stride,
                        uint8_t* codes, uint8_t* sf, float* deq) {
    const int G = cols / 16;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        float gr = g[(int64_t)r * g_stride];
        uint8_t c16[16];
        float d16[16];
        for (int q = 0; q < G; ++q) {
            const float* src = a + (int64_t)r * cols + q * 16;
            nvfp4_group(src, gr, c16, sf + (int64_t)r * G + q, d16);
            pack_group(c16, codes + (int64_t)r * (cols / 2), q);
            if (deq) memcpy(deq + (int64_t)r * cols + q * 16, d16, sizeof d16);
        }
    }
}

/* Dequantize packed codes + scales (fp32 ops: val * fp32(dec(sf) * g)). */
void orc_nvfp4_dequantize(const uint8_t* codes, const uint8_t* sf, int rows, int cols, const float* g,
                          int g_stride, float* out) {
    const int G = cols / 16;
#pragma omp parallel for schedule(static)
    for (int r = 0; r < rows; ++r) {
        float gr = g[(int64_t)r * g_stride];
        for (int k = 0; k < cols; ++k) {
            uint8_t byte = codes[(int64_t)r * (cols / 2) + k / 2];
            uint8_t c = (k & 1) ? (byte >> 4) : (byte & 15);
            float d = (float)orc_e4m3_value(sf[(int64_t)r * G + k / 16]) * gr;
            out[(int64_t)r * cols + k] = (float)orc_e2m1_value(c) * d;
        }
    }
}

/*
 * Weight quantization (A1). Base: NVFP4(W, g_w) with g_w from the whole matrix.
 * Residual: R = fp32(W - deq Q(W)) for every element, quantized to NVFP4 with the
 * same g_w. Both are produced for every block; the block selection comes later.
 */
void orc_quantize_weight(const uint16_t* W, int N, int K, uint8_t* base_codes, uint8_t* base_sf,
                         float* g_w, uint8_t* res_codes, uint8_t* res_sf) {
    const int64_t NK = (int64_t)N * K;
    float* w = (float*)malloc(sizeof(float) * NK);
    float* deq = (float*)malloc(sizeof(float) * NK);
    for (int64_t i = 0; i < NK; ++i) w[i] = bf16_to_f32(W[i]);
    float g = orc_global_scale_f32(w, NK);
    *g_w = g;
    orc_nvfp4_quantize(w, N, K, &g, 0, base_codes, base_sf, deq);
    for (int64_t i = 0; i < NK; ++i) deq[i] = w[i] - deq[i]; /* R, fp32 */
    orc_nvfp4_quantize(deq, N, K, &g, 0, res_codes, res_sf, NULL);
    free(w);
    free(deq);
}

/* Activation quantization (A6): per-token tensor scale g_x[m] = amax(X[m,:]) / 2688
 * (1 for an all-zero row), then NVFP4 of the row with that scale. */
void orc_quantize_act(const uint16_t* X, int M, int K, uint8_t* codes, uint8_t* sf, float* g_x) {
    float* x = (float*)malloc(sizeof(float) * (int64_t)M * K);
    for (int64_t i = 0; i < (int64_t)M * K; ++i) x[i] = bf16_to_f32(X[i]);
    for (int m = 0; m < M; ++m) g_x[m] = orc_global_scale_f32(x + (int64_t)m * K, K);
    orc_nvfp4_quantize(x, M, K, g_x, 1, codes, sf, NULL);
    free(x);
}

/* Diagonal Hessian estimate (A2): H_k = fp32( S_k / T ) with S_k the fp64 sum of the
 * squares fp64(x_tk)^2 (exact: x is bf16) taken by a fixed pairwise tree over t: the T
 * squares padded with zeros to P = the next power of two, then v[i] += v[i + h] for
 * h = P/2, P/4, ..., 1. The pages give the mean of squares and no summation order;
 * the tree is the order the GPU can run in parallel (the same tree as Delta's). */
void orc_hessian_diag(const uint16_t* Xcal, int T, int K, float* H) {
    int P = 1;
    while (P < T) P <<= 1;
    double* v = (double*)malloc(sizeof(double) * P);
    for (int k = 0; k < K; ++k) {
        for (int t = 0; t < P; ++t) {
            double x = t < T ? (double)bf16_to_f32(Xcal[(int64_t)t * K + k]) : 0.0;
            v[t] = x * x;
        }
        for (int h = P / 2; h >= 1; h >>= 1)
            for (int i = 0; i < h; ++i) v[i] = v[i] + v[i + h];
        H[k] = (float)(v[0] / (double)T);
    }
    free(v);
}

/* Pairwise tree over 64 values: v[i] += v[i+32] (i<32), then +16, +8, +4, +2, +1. */
static double tree64(double* v) {
    for (int h = 32; h >= 1; h >>= 1)
        for (int i = 0; i < h; ++i) v[i] = v[i] + v[i + h];
    return v[0];
}

/*
 * Delta-score (A3) for every 64x64 block b = nt*(K/64) + kt: the block's reduction of
 * the H-weighted squared error when its residual is kept (summary, "Methodology",
 * section 2):
 *   e   = R = fp32(W - deq Q(W))            (base quantization error)
 *   e'  = fp32(R - deq R)                   (error left after the residual)
 *   tau = fp64(e)*fp64(e) - fp64(e')*fp64(e')
 *         (both squares are exact in fp64, so the subtraction is the one rounding)
 *   c_k = tree64 over the block's 64 rows of tau, in fp64
 *   p_k = fp64(H_k) * c_k
 *   Delta_b = tree64 over the block's 64 columns of p_k, in fp64
 */
void orc_delta_score(const uint16_t* W, int N, int K, const float* H, const uint8_t* base_codes,
                     const uint8_t* base_sf, float g_w, const uint8_t* res_codes, const uint8_t* res_sf,
                     double* delta) {
    const int64_t NK = (int64_t)N * K;
    float* dq = (float*)malloc(sizeof(float) * NK);
    float* dr = (float*)malloc(sizeof(float) * NK);
    orc_nvfp4_dequantize(base_codes, base_sf, N, K, &g_w, 0, dq);
    orc_nvfp4_dequantize(res_codes, res_sf, N, K, &g_w, 0, dr);
    const int NBr = N / 64, KB = K / 64;
#pragma omp parallel for schedule(static)
    for (int b = 0; b < NBr * KB; ++b) {
        int nt = b / KB, kt = b % KB;
        double p[64], col[64];
        for (int c = 0; c < 64; ++c) {
            int k = kt * 64 + c;
            for (int r = 0; r < 64; ++r) {
                int64_t i = (int64_t)(nt * 64 + r) * K + k;
                float e = bf16_to_f32(W[i]) - dq[i];
                float e2 = e - dr[i];
                double sq = (double)e * (double)e;      /* exact */
                double sq2 = (double)e2 * (double)e2;   /* exact */
                col[r] = sq - sq2;
            }
            p[c] = (double)H[k] * tree64(col);
        }
        delta[b] = tree64(p);
    }
    free(dq);
    free(dr);
}

typedef struct { double d; int32_t b; } scored_t;

static int cmp_scored(const void* x, const void* y) {
    const scored_t* a = (const scored_t*)x;
    const scored_t* c = (const scored_t*)y;
    if (a->d > c->d) return -1; /* Delta descending */
    if (a->d < c->d) return 1;
    return (a->b > c->b) - (a->b < c->b); /* ties: lower block index first */
}

static int cmp_i32(const void* x, const void* y) {
    int32_t a = *(const int32_t*)x, c = *(const int32_t*)y;
    return (a > c) - (a < c);
}

/* Top-K (A4): order all blocks by (Delta descending, b ascending); rank = the first
 * `budget` block indices in that order; sel = the same set in ascending b. */
void orc_topk(const double* delta, int nblk, int budget, int32_t* rank, int32_t* sel) {
    scored_t* v = (scored_t*)malloc(sizeof(scored_t) * (size_t)(nblk > 0 ? nblk : 1));
    for (int b = 0; b < nblk; ++b) { v[b].d = delta[b]; v[b].b = b; }
    qsort(v, (size_t)nblk, sizeof(scored_t), cmp_scored);
    for (int i = 0; i < budget; ++i) rank[i] = sel[i] = v[i].b;
    qsort(sel, (size_t)budget, sizeof(int32_t), cmp_i32);
    free(v);
}

/*
 * Packed residual (A5) from the full residual codes/scales and the ascending list
 * `sel` of selected blocks b = nt*(K/64) + kt:
 *  blk_codes[i]: 2048 bytes, block row r (0..63), packed byte j (0..31, elements
 *    2j, 2j+1 of the block row) at (r/8)*256 + (j/16)*128 + (r%8)*16 + (j%16):
 *    8x16-byte core matrices, K-adjacent ones 128 B apart, 8-row groups 256 B apart.
 *  blk_sf[i]: 512 bytes, the block's scales written into the 128-row scale tile of
 *    the 128-row band holding it: tile row t = 64*(nt%2) + r, group q (0..3) at
 *    (t%32)*16 + (t/32)*4 + q; every other byte zero.
 *  blk_kt[i] = kt;  tile_ptr[nt] = #selected blocks in rows < nt (size N/64 + 1);
 *  bitmap[nt][w] bit j set iff block (nt, 32w + j) is selected, w < ceil((K/64)/32).
 */
void orc_pack_residual(const uint8_t* res_codes, const uint8_t* res_sf, int N, int K, const int32_t* sel,
                       int budget, uint8_t* blk_codes, uint8_t* blk_sf, int32_t* blk_kt, int32_t* tile_ptr,
                       uint32_t* bitmap) {
    const int KB = K / 64, NBr = N / 64, KW = (KB + 31) / 32;
    memset(blk_sf, 0, (size_t)budget * 512);
    memset(bitmap, 0, sizeof(uint32_t) * (size_t)NBr * KW);
    for (int nt = 0; nt <= NBr; ++nt) tile_ptr[nt] = 0;
    for (int i = 0; i < budget; ++i) {
        int b = sel[i], nt = b / KB, kt = b % KB;
        for (int r = 0; r < 64; ++r) {
            const uint8_t* src = res_codes + (int64_t)(nt * 64 + r) * (K / 2) + kt * 32;
            for (int j = 0; j < 32; ++j)
                blk_codes[(int64_t)i * 2048 + (r / 8) * 256 + (j / 16) * 128 + (r % 8) * 16 + (j % 16)] = src[j];
            int t = 64 * (nt % 2) + r;
            for (int q = 0; q < 4; ++q)
                blk_sf[(int64_t)i * 512 + (t % 32) * 16 + (t / 32) * 4 + q] =
                    res_sf[(int64_t)(nt * 64 + r) * (K / 16) + kt * 4 + q];
        }
        blk_kt[i] = kt;
        bitmap[(int64_t)nt * KW + kt / 32] |= 1u << (kt % 32);
        tile_ptr[nt + 1] += 1;
    }
    for (int nt = 0; nt < NBr; ++nt) tile_ptr[nt + 1] += tile_ptr[nt];
}

/*
 * Tiled scale layout consumed by the GEMM. Rows are grouped in tiles of 128 and
 * groups in fours (64 K elements); each (row tile, 64-K step) is one 512-byte
 * chunk, chunks ordered row tile major, K step minor. Inside a chunk, row t of the
 * tile and group q of the step sit at (t%32)*16 + (t/32)*4 + q. Rows beyond `rows`
 * (up to the next multiple of 128) are zero. Size: ceil(rows/128)*128 * (cols/16).
 */
void orc_sf_tile(const uint8_t* sf, int rows, int cols, uint8_t* out) {
    const int G = cols / 16, KS = cols / 64, RT = (rows + 127) / 128;
    memset(out, 0, (size_t)RT * 128 * G);
    for (int r = 0; r < rows; ++r)
        for (int q = 0; q < G; ++q) {
            int t = r % 128;
            int64_t chunk = (int64_t)(r / 128) * KS + q / 4;
            out[chunk * 512 + (t % 32) * 16 + (t / 32) * 4 + (q % 4)] = sf[(int64_t)r * G + q];
        }
}

/*
 * GEMM reference (A7-A8) for a list of output rows:
 *   y[m,n] = g_x[m] * g_w * sum_k xh_mk * (wh_nk + [b(n,k) selected] * rh_nk)
 * with xh = val(cx) * dec(sfx), wh = val(cw) * dec(sfw), rh = val(cr) * dec(sfr)
 * (all exact in fp64), the sum taken sequentially over k in fp64.
 * yabs[m,n] = g_x[m] * g_w * sum_k |xh_mk * (wh_nk + [sel] rh_nk)| (tolerance scale).
 * mode: 0 base + residual, 1 base only, 2 residual only.
 * blk_mask: [N/64][K/64] bytes, nonzero for selected blocks (NULL: none).
 */
void orc_gemm_rows(const uint8_t* x_codes, const uint8_t* x_sf, const float* g_x, const uint8_t* w_codes,
                   const uint8_t* w_sf, float g_w, const uint8_t* r_codes, const uint8_t* r_sf,
                   const uint8_t* blk_mask, int M, int N, int K, int mode, const int32_t* rows, int nrows,
                   double* y, double* yabs) {
    const int G = K / 16, KB = K / 64;
    (void)M;
    double* xh = (double*)malloc(sizeof(double) * (size_t)nrows * K);
    for (int i = 0; i < nrows; ++i) {
        int m = rows[i];
        for (int k = 0; k < K; ++k) {
            uint8_t byte = x_codes[(int64_t)m * (K / 2) + k / 2];
            xh[(int64_t)i * K + k] = orc_e2m1_value((k & 1) ? byte >> 4 : byte & 15) *
                                     orc_e4m3_value(x_sf[(int64_t)m * G + k / 16]);
        }
    }
#pragma omp parallel for schedule(dynamic, 16)
    for (int n = 0; n < N; ++n) {
        double* wh = (double*)malloc(sizeof(double) * K);
        for (int k = 0; k < K; ++k) {
            double v = 0.0;
            if (mode != 2) {
                uint8_t byte = w_codes[(int64_t)n * (K / 2) + k / 2];
                v += orc_e2m1_value((k & 1) ? byte >> 4 : byte & 15) * orc_e4m3_value(w_sf[(int64_t)n * G + k / 16]);
            }
            if (mode != 1 && blk_mask && blk_mask[(int64_t)(n / 64) * KB + k / 64]) {
                uint8_t byte = r_codes[(int64_t)n * (K / 2) + k / 2];
                v += orc_e2m1_value((k & 1) ? byte >> 4 : byte & 15) * orc_e4m3_value(r_sf[(int64_t)n * G + k / 16]);
            }
            wh[k] = v;
        }
        for (int i = 0; i < nrows; ++i) {
            double s = 0.0, sa = 0.0;
            const double* xr = xh + (int64_t)i * K;
            for (int k = 0; k < K; ++k) {
                double t = xr[k] * wh[k];
                s += t;
                sa += fabs(t);
            }
            double scale = (double)g_x[rows[i]] * (double)g_w;
            y[(int64_t)i * N + n] = scale * s;
            if (yabs) yabs[(int64_t)i * N + n] = scale * sa;
        }
        free(wh);
    }
    free(xh);
}

/*
 * Equivalent transform ahead of quantization (MosaicQuant summary, "Methodology",
 * section 1: activation outliers are first migrated into the weights by an equivalent
 * transform such as SmoothQuant). The pages name the transform but do not define it;
 * this is SmoothQuant's per-input-channel rule with migration strength alpha = 1/2:
 *   ax_k = max_t |Xcal[t][k]|,  aw_k = max_n |W[n][k]|,
 *   s_k  = fp32( sqrt( fp32(ax_k / aw_k) ) )   (1 if ax_k or aw_k is 0),
 * so that X W^T = (X diag(s)^-1) (W diag(s))^T, and both sides then peak at
 * sqrt(ax_k * aw_k) in channel k. Division and square root are IEEE, rounded once each.
 */
void orc_smooth_scales(const uint16_t* Xcal, int T, const uint16_t* W, int N, int K, float* s) {
    for (int k = 0; k < K; ++k) {
        float ax = 0.0f, aw = 0.0f;
        for (int t = 0; t < T; ++t) ax = fmaxf(ax, fabsf(bf16_to_f32(Xcal[(int64_t)t * K + k])));
        for (int n = 0; n < N; ++n) aw = fmaxf(aw, fabsf(bf16_to_f32(W[(int64_t)n * K + k])));
        s[k] = (ax == 0.0f || aw == 0.0f) ? 1.0f : sqrtf(ax / aw);
    }
}

/* Round an fp32 value to bf16 (nearest, ties to even; the inputs here are finite). */
static uint16_t f32_to_bf16_rne(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

/* Apply the transform to rows x K bf16 values: out = bf16(a * s_k) for the weight
 * (invert = 0), out = bf16(a / s_k) for activations (invert = 1), one IEEE operation and
 * one rounding to bf16 each. */
void orc_smooth_apply(const uint16_t* A, int rows, int K, const float* s, int invert, uint16_t* out) {
    for (int64_t r = 0; r < rows; ++r)
        for (int k = 0; k < K; ++k) {
            float a = bf16_to_f32(A[r * K + k]);
            out[r * K + k] = f32_to_bf16_rne(invert ? a / s[k] : a * s[k]);
        }
}
