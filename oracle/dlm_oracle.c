/*
 * dlm_oracle.c -- plain, slow, obviously-correct CPU oracle for the
 * diffusion-LM noising-plus-loss path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or
 * calls this file: only the test suite, the smoke check of the package entry
 * point and the CPU-baseline leg of the benchmark use it.  It shares no code,
 * header, table or helper with the CUDA library.
 *
 * Build: gcc -O2 -fopenmp -ffp-contract=off -shared -fPIC (see build.py).
 * -ffp-contract=off matters: the fp32 mask-probability arithmetic must round
 * after every multiply and every add, exactly as written below.
 *
 * What it follows (page title, section):
 *   [LLaDA]   "LLaDA-8B-MDLM-LoRA", Training table, row "Objective":
 *             t ~ U(0,1) per sequence, mask probability (1-1e-3)t + 1e-3,
 *             CE on masked tokens divided by the mask probability.
 *   [Axolotl] "Native diffusion language-model training", model table
 *             (absorbing mask; aligned logits for Nemotron, shifted for
 *             Dream; uniform token noise for DiffusionGemma) and
 *             "Packed training" (documents isolated, positions restart at
 *             document boundaries).
 *   [Gemma]   "diffusiongemma-26B-A4B-it-ALWAYS-THINK", Finetuning notes:
 *             total = diffusion_CE + w * encoder_AR_CE, canvas positions
 *             replaced by uniform-random vocabulary ids at a per-example
 *             rate t ~ U(eps, 1).
 *   [SM64]    Steele, Lea & Flood, "Fast Splittable Pseudorandom Number
 *             Generators", OOPSLA 2014 (SplitMix64: state advances by the
 *             golden gamma 0x9E3779B97F4A7C15, output = mix64 of the state),
 *             with the "variant 13" 64-bit finaliser of D. Stafford,
 *             "Better Bit Mixing" (2011): shifts 30/27/31 and multipliers
 *             0xBF58476D1CE4E5B9, 0x94D049BB133111EB.
 *
 * The pages define no random-number generator; the counter construction
 * (stream, unit, position) -> SplitMix64 output is this library's documented
 * choice, implemented here from the published definition above.
 */
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#include <math.h>

#define DLMO_GAMMA 0x9E3779B97F4A7C15ULL

/* ---------------------------------------------------------------------- */
/* [SM64] the k-th output (k = counter + 1) of a SplitMix64 generator whose
 * initial state is `seed`: state_k = seed + k * gamma (mod 2^64), then the
 * variant-13 finaliser. */
uint64_t dlmo_splitmix64_at(uint64_t seed, uint64_t counter)
{
    uint64_t z = seed + (counter + 1ULL) * DLMO_GAMMA;
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ULL;
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBULL;
    return z ^ (z >> 31);
}

/* Counter layout: stream in bits 56..63, unit in bits 32..55, position within
 * the unit in bits 0..31.  Streams: 0 = time draw, 1 = corruption decision,
 * 2 = replacement id. */
uint64_t dlmo_counter(uint32_t stream, uint32_t unit, uint32_t pos)
{
    return ((uint64_t)stream << 56) | ((uint64_t)unit << 32) | (uint64_t)pos;
}

/* 24 high bits of a draw, as an integer in [0, 2^24). */
static uint32_t u24_of(uint64_t h) { return (uint32_t)(h >> 40); }

/* ---------------------------------------------------------------------- */
/* Time and mask probability per unit.
 *   absorbing [LLaDA]: t = u,                 p = (1 - eps) t + eps
 *   uniform   [Gemma]: t = (1 - eps) u + eps, p = t
 * u = u24 / 2^24 (exact in fp32).  Every operation is one fp32 rounding:
 * c1 = fl(1 - eps), then fl(fl(c1 * x) + eps). */
void dlmo_sample_t(uint64_t seed, int32_t n_units, int32_t mode, float eps,
                   float *t, float *p)
{
    const float c1 = 1.0f - eps;
    for (int32_t u = 0; u < n_units; ++u) {
        uint32_t k = u24_of(dlmo_splitmix64_at(seed, dlmo_counter(0, (uint32_t)u, 0)));
        float x = (float)k * (1.0f / 16777216.0f);
        float scaled = c1 * x;          /* one rounding */
        float v = scaled + eps;         /* one rounding */
        if (mode == 0) { t[u] = x; p[u] = v; }
        else           { t[u] = v; p[u] = v; }
    }
}

/* Unit and within-unit position of token i.  Dense layout: unit = i / L.
 * Packed layout: the unit whose [cu[u], cu[u+1]) holds i ([Axolotl] Packed
 * training: positions restart at document boundaries).  Linear scan -- slow
 * on purpose, obviously right. */
static int locate(int64_t i, int32_t n_units, int32_t seq_len,
                  const int32_t *cu, int32_t *unit, int64_t *pos)
{
    if (!cu) {
        *unit = (int32_t)(i / seq_len);
        *pos = i % seq_len;
        return 0;
    }
    for (int32_t u = 0; u < n_units; ++u) {
        if (i >= cu[u] && i < cu[u + 1]) { *unit = u; *pos = i - cu[u]; return 0; }
    }
    return -1;
}

/* Corruption of clean ids, one token at a time.
 *   corrupted = (float)u24(stream 1) < p_unit * 2^24   (exact fp32 compare)
 *   pads are never corrupted and keep their id.
 *   absorbing [LLaDA]: noisy = mask_id
 *   uniform   [Gemma]: noisy = ((h(stream 2) >> 32) * V) >> 32, a uniform id
 *                      in [0, V); equal to the clean id is allowed.
 * Returns 0, or -1 if the layout is inconsistent. */
int dlmo_corrupt(int32_t n_units, int32_t seq_len, const int32_t *cu_seqlens,
                 const uint8_t *pad_mask, int64_t n_tokens,
                 const int32_t *clean, const float *p, int32_t mode,
                 int32_t mask_id, int32_t vocab, uint64_t seed,
                 int32_t *noisy, uint8_t *corrupted)
{
    for (int64_t i = 0; i < n_tokens; ++i) {
        int32_t u; int64_t pos;
        if (locate(i, n_units, seq_len, cu_seqlens, &u, &pos) != 0) return -1;
        if (pad_mask && pad_mask[i]) { noisy[i] = clean[i]; corrupted[i] = 0; continue; }
        uint64_t h1 = dlmo_splitmix64_at(seed, dlmo_counter(1, (uint32_t)u, (uint32_t)pos));
        float thr = p[u] * 16777216.0f;
        int c = (float)u24_of(h1) < thr;
        corrupted[i] = (uint8_t)c;
        if (!c) { noisy[i] = clean[i]; continue; }
        if (mode == 0) {
            noisy[i] = mask_id;
        } else {
            uint64_t h2 = dlmo_splitmix64_at(seed, dlmo_counter(2, (uint32_t)u, (uint32_t)pos));
            noisy[i] = (int32_t)(((h2 >> 32) * (uint64_t)(uint32_t)vocab) >> 32);
        }
    }
    return 0;
}

/* ---------------------------------------------------------------------- */
/* Cross-entropy of one row, the textbook definition in double:
 *   m = max_v x_v,  lse = m + log sum_v exp(x_v - m),  ce = lse - x_y. */
static double row_lse(const double *x, int32_t V)
{
    double m = x[0];
    for (int32_t v = 1; v < V; ++v) if (x[v] > m) m = x[v];
    double s = 0.0;
    for (int32_t v = 0; v < V; ++v) s += exp(x[v] - m);
    return m + log(s);
}

static double bf16_to_double(uint16_t b)
{
    uint32_t w = (uint32_t)b << 16;
    float f;
    memcpy(&f, &w, sizeof f);
    return (double)f;
}

static void decode_row(const uint16_t *src, int32_t V, double *dst)
{
    for (int32_t v = 0; v < V; ++v) dst[v] = bf16_to_double(src[v]);
}

/* lse and ce for n rows of a bf16 logits matrix (row stride ld elements).
 * Rows are independent; each result lands in its own slot. */
void dlmo_ce_rows_bf16(const uint16_t *logits, int64_t ld, int32_t V, int64_t n,
                       const int64_t *rows, const int32_t *targets,
                       double *lse, double *ce)
{
    #pragma omp parallel
    {
        double *buf = (double *)malloc(sizeof(double) * (size_t)V);
        #pragma omp for schedule(dynamic, 1)
        for (int64_t k = 0; k < n; ++k) {
            decode_row(logits + rows[k] * ld, V, buf);
            double l = row_lse(buf, V);
            lse[k] = l;
            ce[k] = l - buf[targets[k]];
        }
        free(buf);
    }
}

/* Same on a double matrix (used for logits formed as H W^T in double). */
void dlmo_ce_rows_f64(const double *z, int64_t ld, int32_t V, int64_t n,
                      const int64_t *rows, const int32_t *targets,
                      double *lse, double *ce)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t k = 0; k < n; ++k) {
        const double *x = z + rows[k] * ld;
        double l = row_lse(x, V);
        lse[k] = l;
        ce[k] = l - x[targets[k]];
    }
}

/* Gradient of coef * ce with respect to the row's logits:
 *   d[v] = coef * (exp(x_v - lse) - [v == y]). */
void dlmo_grad_rows_bf16(const uint16_t *logits, int64_t ld, int32_t V, int64_t n,
                         const int64_t *rows, const int32_t *targets,
                         const double *coef, const double *lse, double *out)
{
    #pragma omp parallel
    {
        double *buf = (double *)malloc(sizeof(double) * (size_t)V);
        #pragma omp for schedule(dynamic, 1)
        for (int64_t k = 0; k < n; ++k) {
            decode_row(logits + rows[k] * ld, V, buf);
            double *o = out + k * (int64_t)V;
            for (int32_t v = 0; v < V; ++v)
                o[v] = coef[k] * (exp(buf[v] - lse[k]) - (v == targets[k] ? 1.0 : 0.0));
        }
        free(buf);
    }
}

void dlmo_grad_rows_f64(const double *z, int64_t ld, int32_t V, int64_t n,
                        const int64_t *rows, const int32_t *targets,
                        const double *coef, const double *lse, double *out)
{
    #pragma omp parallel for schedule(dynamic, 1)
    for (int64_t k = 0; k < n; ++k) {
        const double *x = z + rows[k] * ld;
        double *o = out + k * (int64_t)V;
        for (int32_t v = 0; v < V; ++v)
            o[v] = coef[k] * (exp(x[v] - lse[k]) - (v == targets[k] ? 1.0 : 0.0));
    }
}

/* Decode a bf16 array to double (test convenience for the linear path). */
void dlmo_bf16_to_f64(const uint16_t *src, int64_t n, double *dst)
{
    #pragma omp parallel for schedule(static)
    for (int64_t i = 0; i < n; ++i) dst[i] = bf16_to_double(src[i]);
}
