/*
 * msa_oracle.c — plain, slow CPU oracle for MiniMax-Sparse-Attention (MSA)
 * decode over an NVFP4 KV cache.
 *
 * TEST INFRASTRUCTURE ONLY.  Only the test suite, the smoke check and the
 * benchmark's CPU-baseline leg may load this library.  It shares no code,
 * header, table or constant with the CUDA path under
 * block_sparse_attention_10_b200/csrc and never calls it.
 *
 * What it computes (all floating-point sums in double, fixed loop order):
 *
 *   Source: "vLLM Adds Day-0 Support for MiniMax-M3.1-Flash on NVIDIA and AMD
 *   GPUs" (ainewsbites.com), section "A model built for efficient inference":
 *   the KV cache is cut into 128-token blocks; a lightweight indexer scores
 *   every key of the context and those scores are pooled into one score per
 *   block; exact attention then runs over the 16 best blocks only, the most
 *   recent block always kept, so at most 2,048 keys per query.  The same
 *   section and the readmex.ai TL;DR say both the indexer keys and the
 *   attention K/V are held in NVFP4.
 *
 * The pages leave the functional forms open; this oracle fixes them as follows
 * (the same readings the CUDA path implements):
 *   - NVFP4: E2M1 codes (sign, 2 exponent bits, 1 mantissa bit, bias 1), one
 *     E4M3 (OCP "FN": bias 7, max 448, no infinities) scale per 16 elements,
 *     one fp32 scale per tensor.  Element 2i in the low nibble of byte i.
 *     decode: v = fp32( e2m1 * e4m3 ) * s_tensor   (one fp32 rounding).
 *     encode: s = E4M3_rne_sat( amax16 / fp32(6 * s_tensor) ),
 *             code = E2M1_rne_sat( x / fp32(s * s_tensor) ), codes 0 if the
 *             denominator is 0.
 *   - indexer: s_j = sum_h w_h * max(0, q_h . k_j), one index key per token
 *     shared by all indexer heads;
 *   - pooling: mean (pool_mode 0) or max (pool_mode 1) of s_j over the
 *     visible tokens of each block; blocks with no visible token: -inf;
 *   - selection: the query's own block r = pos div 128 plus the best
 *     min(15, NB_vis - 1) other visible blocks by (score desc, index asc),
 *     listed ascending, padded with -1;
 *   - attention: softmax(scale * q.k) . v over the selected keys j <= pos,
 *     query head h reading KV head h div (Hq/Hkv).
 *   Positions: sequence b has length L_b, which includes its Tq query tokens;
 *   query t sits at pos_t = L_b - Tq + t and sees keys 0..pos_t.
 */
#include "msa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>

#define ORC_BLOCK 128
#define ORC_TOPK 16

/* ------------------------------------------------------------------------ */
/* E2M1 and E4M3 element formats                                             */
/* ------------------------------------------------------------------------ */

double orc_e2m1_value(uint8_t code)
{
    int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
    /* bias 1; exponent field 0 is subnormal with the same scale as field 1 */
    double mag = (e == 0) ? ldexp((double)m, -1) : ldexp(1.0 + 0.5 * m, e - 1);
    return s ? -mag : mag;
}

double orc_e4m3_value(uint8_t code)
{
    int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
    double mag;
    if (e == 15 && m == 7)
        return NAN; /* the only non-finite encoding of the FN variant */
    if (e == 0)
        mag = ldexp((double)m, -9); /* (m/8) * 2^(1-7) */
    else
        mag = ldexp(1.0 + m / 8.0, e - 7);
    return s ? -mag : mag;
}

/* Round |x| to a grid with `mbits` mantissa bits, minimum normal exponent
 * `emin`, round to nearest, ties to even (the grid value with the even
 * integer multiple of the quantum). */
static double round_to_grid(double a, int mbits, int emin)
{
    int e2;
    if (a == 0.0)
        return 0.0;
    frexp(a, &e2);           /* a = f * 2^e2, f in [0.5, 1) */
    int E = e2 - 1;          /* a in [2^E, 2^(E+1)) */
    if (E < emin)
        E = emin;            /* subnormal range shares the quantum of emin */
    double q = ldexp(1.0, E - mbits);
    return nearbyint(a / q) * q; /* a/q exact (power of two); nearbyint = RNE */
}

uint8_t orc_e4m3_encode(float xf)
{
    double x = xf;
    uint8_t sign = signbit(x) ? 0x80 : 0x00;
    double a = fabs(x);
    if (isnan(x))
        return 0x7F;
    if (a >= 448.0)
        return sign | 0x7E; /* saturate to the largest finite value */
    double v = round_to_grid(a, 3, -6);
    if (v >= 448.0)
        return sign | 0x7E;
    if (v == 0.0)
        return sign;
    int e2;
    frexp(v, &e2);
    int E = e2 - 1;
    if (E < -6) /* subnormal: v = m * 2^-9 */
        return sign | (uint8_t)(int)ldexp(v, 9);
    int m = (int)((ldexp(v, -E) - 1.0) * 8.0);
    return sign | (uint8_t)(((E + 7) << 3) | m);
}

uint8_t orc_e2m1_encode(float xf)
{
    double x = xf;
    uint8_t sign = signbit(x) ? 0x8 : 0x0;
    double a = fabs(x);
    if (isnan(x))
        return 0x0;
    if (a >= 6.0)
        return sign | 0x7;
    double v = round_to_grid(a, 1, 0);
    if (v >= 6.0)
        return sign | 0x7;
    if (v == 0.0)
        return sign;
    if (v < 1.0) /* subnormal 0.5 */
        return sign | 0x1;
    int e2;
    frexp(v, &e2);
    int E = e2 - 1;
    int m = (int)((ldexp(v, -E) - 1.0) * 2.0);
    return sign | (uint8_t)(((E + 1) << 1) | m);
}

/* ------------------------------------------------------------------------ */
/* NVFP4 vectors                                                             */
/* ------------------------------------------------------------------------ */

float orc_tensor_scale(const float* x, int64_t n)
{
    float amax = 0.0f;
    for (int64_t i = 0; i < n; ++i) {
        float a = fabsf(x[i]);
        if (a > amax)
            amax = a;
    }
    volatile float denom = 6.0f * 448.0f;
    return amax / denom;
}

void orc_nvfp4_encode(const float* x, int64_t nvec, int dim, float s_tensor,
                      uint8_t* data, uint8_t* scale)
{
    volatile float six_st = 6.0f * s_tensor;
#pragma omp parallel for schedule(static)
    for (int64_t v = 0; v < nvec; ++v) {
        const float* xv = x + v * dim;
        uint8_t* dv = data + v * (dim / 2);
        uint8_t* sv = scale + v * (dim / 16);
        memset(dv, 0, (size_t)(dim / 2));
        for (int g = 0; g < dim / 16; ++g) {
            float amax = 0.0f;
            for (int i = 0; i < 16; ++i) {
                float a = fabsf(xv[g * 16 + i]);
                if (a > amax)
                    amax = a;
            }
            volatile float ratio = amax / six_st;
            uint8_t sc = orc_e4m3_encode(ratio);
            sv[g] = sc;
            volatile float denom = (float)orc_e4m3_value(sc) * s_tensor;
            for (int i = 0; i < 16; ++i) {
                int d = g * 16 + i;
                uint8_t c = 0;
                if (denom != 0.0f) {
                    volatile float y = xv[d] / denom;
                    c = orc_e2m1_encode(y);
                }
                dv[d / 2] |= (uint8_t)((d & 1) ? (c << 4) : c);
            }
        }
    }
}

/* Decoded element d of vector `v` of an NVFP4 plane pair. */
static inline float nvfp4_elem(const uint8_t* data, const uint8_t* scale, int dim,
                               float s_tensor, int64_t v, int d)
{
    uint8_t byte = data[v * (dim / 2) + d / 2];
    uint8_t code = (d & 1) ? (byte >> 4) : (byte & 0xF);
    uint8_t sc = scale[v * (dim / 16) + d / 16];
    volatile float p = (float)(orc_e2m1_value(code) * orc_e4m3_value(sc)); /* exact */
    volatile float r = p * s_tensor;
    return r;
}

void orc_nvfp4_decode(const uint8_t* data, const uint8_t* scale, int64_t nvec, int dim,
                      float s_tensor, float* out)
{
#pragma omp parallel for schedule(static)
    for (int64_t v = 0; v < nvec; ++v)
        for (int d = 0; d < dim; ++d)
            out[v * dim + d] = nvfp4_elem(data, scale, dim, s_tensor, v, d);
}

/* Vector (b, h, j) of a cache laid out [B][heads][lmax][...]. */
static inline int64_t cache_vec(const orc_nvfp4* c, int b, int h, int64_t j)
{
    return ((int64_t)b * c->heads + h) * c->lmax + j;
}

/* ------------------------------------------------------------------------ */
/* Indexer + block pooling                                                   */
/* ------------------------------------------------------------------------ */

void orc_index(int B, int Tq, int HI, int DI, const int32_t* seq_lens,
               const float* q_idx, const float* w_idx, const orc_nvfp4* ik,
               int pool_mode, double* token_scores, double* block_scores)
{
    const int64_t lmax = ik->lmax;
    const int64_t nbmax = (lmax + ORC_BLOCK - 1) / ORC_BLOCK;
#pragma omp parallel for collapse(2) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < Tq; ++t) {
            const int64_t L = seq_lens[b];
            const int64_t pos = L - Tq + t;
            const float* q = q_idx + ((int64_t)b * Tq + t) * HI * DI;
            double* ts = token_scores ? token_scores + ((int64_t)b * Tq + t) * lmax : NULL;
            double* bs = block_scores + ((int64_t)b * Tq + t) * nbmax;
            float* kd = (float*)malloc(sizeof(float) * (size_t)DI);
            for (int64_t n = 0; n < nbmax; ++n)
                bs[n] = -INFINITY;
            double acc = 0.0;
            int64_t cnt = 0;
            for (int64_t j = 0; j <= pos; ++j) {
                int64_t vec = cache_vec(ik, b, 0, j);
                for (int d = 0; d < DI; ++d)
                    kd[d] = nvfp4_elem(ik->data, ik->scale, DI, ik->tensor_scale, vec, d);
                double s = 0.0;
                for (int h = 0; h < HI; ++h) {
                    double dot = 0.0;
                    for (int d = 0; d < DI; ++d)
                        dot += (double)q[h * DI + d] * (double)kd[d];
                    double wh = w_idx ? (double)w_idx[((int64_t)b * Tq + t) * HI + h] : 1.0;
                    s += wh * (dot > 0.0 ? dot : 0.0);
                }
                if (ts)
                    ts[j] = s;
                /* pool over the visible tokens of block j / 128 */
                if (pool_mode == 1)
                    acc = (cnt == 0 || s > acc) ? s : acc;
                else
                    acc += s;
                cnt += 1;
                if ((j + 1) % ORC_BLOCK == 0 || j == pos) {
                    bs[j / ORC_BLOCK] = pool_mode == 1 ? acc : acc / (double)cnt;
                    acc = 0.0;
                    cnt = 0;
                }
            }
            free(kd);
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Top-16 block selection with the recent block forced                       */
/* ------------------------------------------------------------------------ */

/* (score desc, index asc): a before b? */
static int ranks_before(double sa, int64_t ia, double sb, int64_t ib)
{
    if (sa > sb) return 1;
    if (sa < sb) return 0;
    return ia < ib;
}

void orc_select(int B, int Tq, int64_t nbmax, const int32_t* seq_lens,
                const double* block_scores, int32_t* sel)
{
#pragma omp parallel for collapse(2) schedule(static)
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < Tq; ++t) {
            const int64_t pos = (int64_t)seq_lens[b] - Tq + t;
            const int64_t r = pos / ORC_BLOCK;           /* forced: the query's own block */
            const int64_t nvis = r + 1;
            const double* s = block_scores + ((int64_t)b * Tq + t) * nbmax;
            int32_t* out = sel + ((int64_t)b * Tq + t) * ORC_TOPK;
            int64_t chosen[ORC_TOPK];
            int nch = 0;
            chosen[nch++] = r;
            int64_t want = nvis - 1 < ORC_TOPK - 1 ? nvis - 1 : ORC_TOPK - 1;
            /* selection by repeated arg-best over the not-yet-chosen blocks */
            for (int64_t k = 0; k < want; ++k) {
                int64_t best = -1;
                for (int64_t n = 0; n < nvis; ++n) {
                    int taken = 0;
                    for (int c = 0; c < nch; ++c)
                        taken |= (chosen[c] == n);
                    if (taken)
                        continue;
                    if (best < 0 || ranks_before(s[n], n, s[best], best))
                        best = n;
                }
                chosen[nch++] = best;
            }
            /* ascending order */
            for (int i = 1; i < nch; ++i)
                for (int j = i; j > 0 && chosen[j - 1] > chosen[j]; --j) {
                    int64_t tmp = chosen[j];
                    chosen[j] = chosen[j - 1];
                    chosen[j - 1] = tmp;
                }
            for (int i = 0; i < ORC_TOPK; ++i)
                out[i] = i < nch ? (int32_t)chosen[i] : -1;
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Exact softmax attention over the selected keys                            */
/* ------------------------------------------------------------------------ */

void orc_attend(int B, int Tq, int Hq, int Hkv, int D, const int32_t* seq_lens,
                const float* q, const orc_nvfp4* k, const orc_nvfp4* v,
                const int32_t* sel, double scale, double* out, double* lse)
{
    const int g = Hq / Hkv;
#pragma omp parallel for collapse(3) schedule(dynamic)
    for (int b = 0; b < B; ++b) {
        for (int t = 0; t < Tq; ++t) {
            for (int h = 0; h < Hq; ++h) {
                const int64_t pos = (int64_t)seq_lens[b] - Tq + t;
                const int hk = h / g;
                const float* qh = q + (((int64_t)b * Tq + t) * Hq + h) * D;
                const int32_t* sl = sel + ((int64_t)b * Tq + t) * ORC_TOPK;
                double* o = out + (((int64_t)b * Tq + t) * Hq + h) * D;
                /* gather the visible selected keys */
                int64_t keys[ORC_TOPK * ORC_BLOCK];
                int nk = 0;
                for (int i = 0; i < ORC_TOPK; ++i) {
                    if (sl[i] < 0)
                        continue;
                    for (int64_t j = (int64_t)sl[i] * ORC_BLOCK; j < (int64_t)(sl[i] + 1) * ORC_BLOCK; ++j)
                        if (j <= pos)
                            keys[nk++] = j;
                }
                double* sc = (double*)malloc(sizeof(double) * (size_t)(nk > 0 ? nk : 1));
                double mx = -INFINITY;
                for (int i = 0; i < nk; ++i) {
                    int64_t vec = cache_vec(k, b, hk, keys[i]);
                    double dot = 0.0;
                    for (int d = 0; d < D; ++d)
                        dot += (double)qh[d] * (double)nvfp4_elem(k->data, k->scale, D, k->tensor_scale, vec, d);
                    sc[i] = dot * scale;
                    if (sc[i] > mx)
                        mx = sc[i];
                }
                double l = 0.0;
                for (int d = 0; d < D; ++d)
                    o[d] = 0.0;
                for (int i = 0; i < nk; ++i) {
                    double p = exp(sc[i] - mx);
                    l += p;
                    int64_t vec = cache_vec(v, b, hk, keys[i]);
                    for (int d = 0; d < D; ++d)
                        o[d] += p * (double)nvfp4_elem(v->data, v->scale, D, v->tensor_scale, vec, d);
                }
                for (int d = 0; d < D; ++d)
                    o[d] = nk > 0 ? o[d] / l : 0.0;
                if (lse)
                    lse[((int64_t)b * Tq + t) * Hq + h] = nk > 0 ? mx + log(l) : -INFINITY;
                free(sc);
            }
        }
    }
}

int orc_num_threads(void)
{
#ifdef _OPENMP
    extern int omp_get_max_threads(void);
    return omp_get_max_threads();
#else
    return 1;
#endif
}
