/*
 * Seeded, counter-based synthetic inputs for the MosaicQuant / ZipperEngine path.
 *
 * This file generates numbers only: Gaussian weights and activations with
 * planted outliers, rounded to bf16. It holds none of the quantization, scoring
 * or GEMM arithmetic; the CPU oracle and the CUDA library both read the bytes it
 * writes, so neither can influence the other through it.
 *
 * Generator: SplitMix64 (Steele, Lea & Flood, "Fast splittable pseudorandom
 * number generators", OOPSLA 2014) used in counter form: the i-th draw of stream
 * `seed` is mix(s0 + (i + 1) * GOLDEN) with s0 = mix(seed + GOLDEN). Uniforms take
 * the top 53 bits; normals use the cosine branch of the Box-Muller transform.
 *
 * Workload shapes follow the pages' model families (LLaMA3 and Qwen3 layers):
 * weights ~ N(0, sigma^2) with a fraction of entries multiplied by a large factor
 * inside a subset of 64x64 blocks (the block-concentrated error the method
 * targets), activations ~ N(0, 1) with a few input channels scaled up.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define GOLDEN 0x9E3779B97F4A7C15ull

static inline uint64_t mix64(uint64_t z) {
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
}

/* i-th 64-bit draw of stream `seed`. */
uint64_t synth_draw(uint64_t seed, uint64_t i) {
    uint64_t s0 = mix64(seed + GOLDEN);
    return mix64(s0 + (i + 1) * GOLDEN);
}

static inline double unif53(uint64_t x) { return (double)(x >> 11) * (1.0 / 9007199254740992.0); }

/* i-th standard normal of stream `seed`. */
double synth_normal(uint64_t seed, uint64_t i) {
    double u1 = unif53(synth_draw(seed, 2 * i));
    double u2 = unif53(synth_draw(seed, 2 * i + 1));
    return sqrt(-2.0 * log(1.0 - u1)) * cos(6.283185307179586476925286766559 * u2);
}

/* fp32 -> bf16 bits, round to nearest even (inputs are finite). */
static inline uint16_t f32_to_bf16(float f) {
    uint32_t u;
    memcpy(&u, &f, 4);
    uint32_t lsb = (u >> 16) & 1u;
    u += 0x7FFFu + lsb;
    return (uint16_t)(u >> 16);
}

typedef struct { uint64_t key; int64_t idx; } keyed_t;

static int cmp_keyed(const void* a, const void* b) {
    const keyed_t* x = (const keyed_t*)a;
    const keyed_t* y = (const keyed_t*)b;
    if (x->key != y->key) return x->key < y->key ? -1 : 1;
    return x->idx < y->idx ? -1 : (x->idx > y->idx);
}

static int cmp_i64(const void* a, const void* b) {
    int64_t x = *(const int64_t*)a, y = *(const int64_t*)b;
    return (x > y) - (x < y);
}

/* Choose `k` distinct indices out of [0, n): the k smallest draws of stream `seed`
 * (ties by index). Writes them ascending into out[k]. Returns 0, or -1 on OOM. */
int synth_choose(uint64_t seed, int64_t n, int64_t k, int64_t* out) {
    if (k <= 0) return 0;
    if (k > n) k = n;
    keyed_t* v = (keyed_t*)malloc(sizeof(keyed_t) * (size_t)n);
    if (!v) return -1;
    for (int64_t i = 0; i < n; ++i) { v[i].key = synth_draw(seed, (uint64_t)i); v[i].idx = i; }
    qsort(v, (size_t)n, sizeof(keyed_t), cmp_keyed);
    for (int64_t i = 0; i < k; ++i) out[i] = v[i].idx;
    free(v);
    qsort(out, (size_t)k, sizeof(int64_t), cmp_i64); /* ascending, for reproducible iteration */
    return 0;
}

/*
 * Weight matrix W[N][K] (bf16 bits): sigma * z, with `n_out` entries multiplied by
 * `mult`. The outliers sit inside `n_out_blocks` of the (N/64)*(K/64) blocks of
 * 64x64 (chosen by stream seed_o), at distinct positions drawn uniformly inside
 * those blocks (stream seed_o + 1). n_out_blocks <= 0 spreads them over the
 * whole matrix. Returns 0 on success.
 */
int synth_weight(uint64_t seed_w, uint64_t seed_o, int N, int K, double sigma,
                 int64_t n_out, int64_t n_out_blocks, double mult, uint16_t* W) {
    const int64_t NK = (int64_t)N * K;
    const int64_t KB = K / 64, NB = (int64_t)(N / 64) * KB;
    unsigned char* is_out = (unsigned char*)calloc((size_t)NK, 1);
    if (!is_out) return -1;
    if (n_out > 0) {
        int64_t* pos = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_out);
        if (!pos) { free(is_out); return -1; }
        if (n_out_blocks > 0 && n_out_blocks < NB) {
            int64_t* blks = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_out_blocks);
            if (!blks) { free(pos); free(is_out); return -1; }
            if (synth_choose(seed_o, NB, n_out_blocks, blks)) { free(blks); free(pos); free(is_out); return -1; }
            int64_t npos = n_out_blocks * 4096;
            if (n_out > npos) n_out = npos;
            if (synth_choose(seed_o + 1, npos, n_out, pos)) { free(blks); free(pos); free(is_out); return -1; }
            for (int64_t i = 0; i < n_out; ++i) {
                int64_t b = blks[pos[i] / 4096], e = pos[i] % 4096;
                int64_t nt = b / KB, kt = b % KB;
                int64_t n = nt * 64 + e / 64, k = kt * 64 + e % 64;
                is_out[n * K + k] = 1;
            }
            free(blks);
        } else {
            if (n_out > NK) n_out = NK;
            if (synth_choose(seed_o + 1, NK, n_out, pos)) { free(pos); free(is_out); return -1; }
            for (int64_t i = 0; i < n_out; ++i) is_out[pos[i]] = 1;
        }
        free(pos);
    }
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < NK; ++i) {
        double v = sigma * synth_normal(seed_w, (uint64_t)i);
        if (is_out[i]) v *= mult;
        W[i] = f32_to_bf16((float)v);
    }
    free(is_out);
    return 0;
}

/*
 * Activations X[M][K] (bf16 bits): z, with the `n_ch` input channels chosen by
 * stream seed_c multiplied by `mult` (the same channels for every token, so the
 * same seed_c gives the same channels in X and in the calibration tokens).
 */
int synth_act(uint64_t seed_x, uint64_t seed_c, int M, int K, int64_t n_ch, double mult, uint16_t* X) {
    unsigned char* hot = (unsigned char*)calloc((size_t)K, 1);
    if (!hot) return -1;
    if (n_ch > 0) {
        int64_t* ch = (int64_t*)malloc(sizeof(int64_t) * (size_t)n_ch);
        if (!ch) { free(hot); return -1; }
        if (synth_choose(seed_c + 7, K, n_ch, ch)) { free(ch); free(hot); return -1; }
        for (int64_t i = 0; i < n_ch; ++i) hot[ch[i]] = 1;
        free(ch);
    }
    const int64_t MK = (int64_t)M * K;
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < MK; ++i) {
        double v = synth_normal(seed_x, (uint64_t)i);
        if (hot[i % K]) v *= mult;
        X[i] = f32_to_bf16((float)v);
    }
    free(hot);
    return 0;
}

/* Plain i.i.d. N(0, sigma^2) bf16 buffer (edge-case tests). */
void synth_normal_bf16(uint64_t seed, double sigma, int64_t n, uint16_t* out) {
#pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) out[i] = f32_to_bf16((float)(sigma * synth_normal(seed, (uint64_t)i)));
}
