/*
 * dsa_oracle.c -- fp64 reference for the DeepSeek Sparse Attention (DSA) hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing in the product path links, loads or calls
 * this file; only the tests, the smoke check and the benchmark's CPU-baseline
 * leg do.  It shares no code, header or table with the CUDA library.
 *
 * Every function is the plain definition written out as loops in double
 * precision, one query row at a time, so that it can be checked by eye against
 * the pages it cites:
 *
 *   [Sel]  "DeepSeek-V3.2-Exp - Keep top-k positions" (Atlas page): the
 *          Indexer.forward listing (model.py 457-487) and the M^sel formula.
 *   [Mask] "DeepSeek-V3.2-Exp - Apply sparse mask" (Atlas page): the MQA
 *          decode listing (model.py 590-606) and S~ = S' + M^sel.
 *   [MLX]  "[WIP] deepseek v32" (ml-explore/mlx-lm PR #512): the fixed indexer
 *          (ReLU, then per-head weight, then the sum over heads).
 *   [Cost] "DeepseekV3.2 lightning indexer design" (llama.cpp discussion
 *          #17692): per cached token the indexer costs 64*128 and MLA 128*576.
 *
 * Data conventions (shared with the CUDA path only through the bytes the
 * seeded input module produces):
 *   - bf16 values arrive as uint16 bit patterns, e4m3 values as uint8 codes;
 *     both are decoded here to double exactly.
 *   - Sequence b owns cache rows [off[b], off[b+1]); E_b = off[b+1]-off[b];
 *     its T query rows sit at absolute positions start_b + t, start_b = E_b - T.
 *   - A query row is r = b*T + t.  Every function takes an optional list of
 *     rows (NULL = all rows, in order); outputs are packed by list position.
 *
 * Build: gcc -O2 -fopenmp -shared -fPIC dsa_oracle.c -o liboracle.so -lm
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

#define OR_HI 64   /* indexer heads  (index_n_heads = 64, MaxText config diff)  */
#define OR_DI 128  /* indexer dim    (index_head_dim = 128)                      */
#define OR_DQK 576 /* latent 512 + rope 64, the absorbed q/k width               */
#define OR_DV 512  /* latent width; the decode listing uses kv_cache as values   */

enum { OR_OK = 0, OR_EINVAL = 1 };

/* ---- exact decoders ---------------------------------------------------- */

double oracle_bf16_to_f64(uint16_t b) {
    uint32_t u = (uint32_t)b << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* OCP e4m3 ("fn" variant): bias 7, no infinities, S.1111.111 is NaN. */
double oracle_e4m3_to_f64(uint8_t v) {
    int s = v >> 7, e = (v >> 3) & 15, m = v & 7;
    double mag;
    if (e == 15 && m == 7) return NAN;
    if (e == 0)
        mag = ldexp((double)m, -9);          /* (m/8) * 2^(1-7) */
    else
        mag = ldexp((double)(8 + m), e - 10); /* (1 + m/8) * 2^(e-7) */
    return s ? -mag : mag;
}

/* ---- act_quant: block-128 e4m3 quantisation ----------------------------
 * [Sel] Indexer.forward quantises q and k with act_quant(x, block_size,
 * scale_fmt) before fp8_index and writes k_cache[start:end] = k_fp8 (its
 * scale kept beside it).  The pages do not print act_quant.  Reading taken:
 * one block = one 128-element vector; scale = amax / 448 in fp32 (1 when
 * amax = 0); each code is the e4m3 value nearest to x / scale (fp32
 * division), ties to the even code, saturating at +-448.  Codes are found
 * from the value table the decoder above defines, not from bit tricks. */

static float e4m3_pos_value(int code) { return (float)oracle_e4m3_to_f64((uint8_t)code); }

uint8_t oracle_e4m3_encode(float x) {
    if (x != x) return 0x7F;
    const uint8_t sign = signbit(x) ? 0x80 : 0x00;
    const float a = fabsf(x);
    if (a >= 448.0f) return sign | 0x7E;  /* 0x7E = 448, the largest finite value */
    int lo = 0;                           /* largest code whose value is <= a     */
    for (int c = 1; c <= 0x7E; ++c)
        if (e4m3_pos_value(c) <= a) lo = c;
    const double vlo = e4m3_pos_value(lo), vhi = e4m3_pos_value(lo + 1);
    const double dlo = (double)a - vlo, dhi = vhi - (double)a;
    int c;
    if (dlo < dhi) c = lo;
    else if (dhi < dlo) c = lo + 1;
    else c = (lo & 1) == 0 ? lo : lo + 1; /* tie: the even code */
    return sign | (uint8_t)c;
}

/* Quantises n_blocks consecutive 128-element bf16 vectors. */
int oracle_quantize_blocks(const uint16_t* x, int64_t n_blocks, uint8_t* codes, float* scales) {
    if (!x || !codes || !scales || n_blocks < 0) return OR_EINVAL;
    for (int64_t i = 0; i < n_blocks; ++i) {
        const uint16_t* xb = x + i * OR_DI;
        float amax = 0.0f;
        for (int d = 0; d < OR_DI; ++d) {
            const float v = fabsf((float)oracle_bf16_to_f64(xb[d]));
            if (v > amax) amax = v;
        }
        const float scale = amax > 0.0f ? amax / 448.0f : 1.0f;
        for (int d = 0; d < OR_DI; ++d)
            codes[i * OR_DI + d] = oracle_e4m3_encode((float)oracle_bf16_to_f64(xb[d]) / scale);
        scales[i] = scale;
    }
    return OR_OK;
}

static void row_geometry(const int32_t* off, int T, int64_t r, int* b, int* t,
                         int64_t* E, int64_t* t_abs) {
    *b = (int)(r / T);
    *t = (int)(r % T);
    *E = (int64_t)off[*b + 1] - off[*b];
    *t_abs = *E - T + *t;
}

static int check_common(const int32_t* off, int B, int T, const int64_t* rows, int64_t n_rows) {
    if (!off || B <= 0 || T <= 0 || n_rows < 0) return OR_EINVAL;
    for (int b = 0; b < B; ++b)
        if (off[b + 1] - off[b] < T) return OR_EINVAL;
    if (rows)
        for (int64_t i = 0; i < n_rows; ++i)
            if (rows[i] < 0 || rows[i] >= (int64_t)B * T) return OR_EINVAL;
    return OR_OK;
}

/* ---- 1. lightning-indexer scores --------------------------------------- */
/*
 * I[t,s] = sum_h w[t,h] * ReLU(q_I[t,h,:] . k_I[s,:])             [MLX], [Sel]
 * plus the causal mask: position s is valid iff s <= start + t; invalid
 * positions get -inf ("index_score += mask", [Sel]).  Positions s >= E are
 * outside the cache and are not written.
 * e4m3 caches (dtype 1): q and k are e4m3 codes, w already carries the q scale,
 * and each key's product is multiplied by its k_scale (the fp8_index call in
 * [Sel] takes k_scale_cache beside the codes).  Scales are positive, so the
 * factor may sit inside or outside the ReLU.
 * mac_count (optional) receives the number of multiply-adds executed.
 */
int oracle_indexer_scores(const void* q_idx, const float* w, const void* k_idx,
                          const float* k_scale, int dtype, const int32_t* off,
                          int B, int T, const int64_t* rows, int64_t n_rows,
                          double* out, int64_t ld, int64_t* mac_count) {
    if (!q_idx || !w || !k_idx || !out || (dtype != 0 && dtype != 1)) return OR_EINVAL;
    if (dtype == 1 && !k_scale) return OR_EINVAL;
    if (!rows) n_rows = (int64_t)B * T;
    if (check_common(off, B, T, rows, n_rows)) return OR_EINVAL;
    int64_t macs = 0;
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t r = rows ? rows[i] : i;
        int b, t;
        int64_t E, t_abs;
        row_geometry(off, T, r, &b, &t, &E, &t_abs);
        if (E > ld) return OR_EINVAL;
        double q[OR_HI][OR_DI];
        for (int h = 0; h < OR_HI; ++h)
            for (int d = 0; d < OR_DI; ++d) {
                int64_t at = (r * OR_HI + h) * OR_DI + d;
                q[h][d] = dtype == 0 ? oracle_bf16_to_f64(((const uint16_t*)q_idx)[at])
                                     : oracle_e4m3_to_f64(((const uint8_t*)q_idx)[at]);
            }
        double wr[OR_HI];
        for (int h = 0; h < OR_HI; ++h) wr[h] = (double)w[r * OR_HI + h];
        double* o = out + i * ld;
        int64_t row_macs = 0;
#pragma omp parallel for schedule(static) reduction(+ : row_macs)
        for (int64_t s = 0; s < E; ++s) {
            if (s > t_abs) {
                o[s] = -INFINITY;
                continue;
            }
            double k[OR_DI];
            int64_t key = (int64_t)off[b] + s;
            for (int d = 0; d < OR_DI; ++d)
                k[d] = dtype == 0 ? oracle_bf16_to_f64(((const uint16_t*)k_idx)[key * OR_DI + d])
                                  : oracle_e4m3_to_f64(((const uint8_t*)k_idx)[key * OR_DI + d]);
            double ks = dtype == 0 ? 1.0 : (double)k_scale[key];
            double score = 0.0;
            for (int h = 0; h < OR_HI; ++h) {
                double dot = 0.0;
                for (int d = 0; d < OR_DI; ++d) dot += q[h][d] * k[d];
                row_macs += OR_DI;
                double relu = dot > 0.0 ? dot : 0.0;
                score += wr[h] * relu * ks;
            }
            o[s] = score;
        }
        macs += row_macs;
    }
    if (mac_count) *mac_count = macs;
    return OR_OK;
}

/* ---- 2. top-k selection ------------------------------------------------ */
/*
 * topk(min(index_topk, end_pos)) over the masked scores ([Sel]): keep each
 * query's k highest-scoring valid positions.  Readings fixed for this build:
 *   - ties: larger score first, then lower position;  -0.0 equals +0.0;
 *   - masked positions (s > start + t) are never kept, so a row keeps
 *     k_eff = min(k, number of valid positions) entries;
 *   - the kept set is written in ascending position order, padded with -1.
 * The scores are read as doubles; a float32 score tensor converted to double
 * keeps its order and its ties exactly.
 */
typedef struct {
    double v;
    int64_t s;
} or_pair;

static int cmp_desc(const void* a, const void* b) {
    const or_pair* x = (const or_pair*)a;
    const or_pair* y = (const or_pair*)b;
    if (x->v > y->v) return -1;
    if (x->v < y->v) return 1;
    return (x->s > y->s) - (x->s < y->s);
}

static int cmp_i32(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x > y) - (x < y);
}

int oracle_topk(const double* scores, int64_t ld, const int32_t* off, int B, int T, int k,
                const int64_t* rows, int64_t n_rows, int32_t* out) {
    if (!scores || !out || k <= 0) return OR_EINVAL;
    if (!rows) n_rows = (int64_t)B * T;
    if (check_common(off, B, T, rows, n_rows)) return OR_EINVAL;
    int bad = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(| : bad)
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t r = rows ? rows[i] : i;
        int b, t;
        int64_t E, t_abs;
        row_geometry(off, T, r, &b, &t, &E, &t_abs);
        if (E > ld) {
            bad = 1;
            continue;
        }
        const double* sc = scores + i * ld;
        int64_t n_valid = 0;
        or_pair* cand = (or_pair*)malloc(sizeof(or_pair) * (size_t)(E > 0 ? E : 1));
        for (int64_t s = 0; s < E; ++s)
            if (s <= t_abs) {
                cand[n_valid].v = sc[s] == 0.0 ? 0.0 : sc[s]; /* -0 -> +0 */
                cand[n_valid].s = s;
                ++n_valid;
            }
        qsort(cand, (size_t)n_valid, sizeof(or_pair), cmp_desc);
        int64_t k_eff = n_valid < k ? n_valid : k;
        int32_t* o = out + i * (int64_t)k;
        for (int64_t j = 0; j < k_eff; ++j) o[j] = (int32_t)cand[j].s;
        qsort(o, (size_t)k_eff, sizeof(int32_t), cmp_i32);
        for (int64_t j = k_eff; j < k; ++j) o[j] = -1;
        free(cand);
    }
    return bad ? OR_EINVAL : OR_OK;
}

/* ---- 3. absorbed MLA over the selected latent rows --------------------- */
/*
 * MQA decode branch, absorbed form ([Mask]):
 *   scores[h,j] = (q_nope[h,:512] . kv[j,:512] + q_pe[h,:] . pe[j,:]) * scale
 *              = scale * q[h,:576] . row_j[:576]     (row = latent || rope)
 *   S~ = S' + M^sel: only the selected positions keep a finite score;
 *   p = softmax_j(S~);  o[h,:] = sum_j p[h,j] * kv[j,:512].
 * The output stays in the 512-wide latent (the wkv_b up-projection that follows
 * in the listing needs trained weights and is outside this path).
 * indices: [n_rows, k] per list position, sequence-local, -1 = empty slot.
 * lse (optional) = natural-log log-sum-exp of the scaled scores per (row, head).
 * A row with no selected position gets o = 0 and lse = -inf.
 */
int oracle_sparse_mla(const uint16_t* q, const uint16_t* kv, const int32_t* off,
                      const int32_t* indices, int B, int T, int H, int k, double scale,
                      const int64_t* rows, int64_t n_rows, double* out, double* lse,
                      int64_t* mac_count) {
    if (!q || !kv || !indices || !out || H <= 0 || k <= 0) return OR_EINVAL;
    if (!rows) n_rows = (int64_t)B * T;
    if (check_common(off, B, T, rows, n_rows)) return OR_EINVAL;
    for (int64_t i = 0; i < n_rows; ++i) {
        int64_t r = rows ? rows[i] : i;
        int64_t E = (int64_t)off[r / T + 1] - off[r / T];
        for (int j = 0; j < k; ++j) {
            int32_t s = indices[i * k + j];
            if (s < -1 || s >= E) return OR_EINVAL;
        }
    }
    int64_t macs = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : macs)
    for (int64_t ih = 0; ih < n_rows * H; ++ih) {
        int64_t i = ih / H;
        int h = (int)(ih % H);
        int64_t r = rows ? rows[i] : i;
        int b = (int)(r / T);
        const int32_t* sel = indices + i * k;
        double qh[OR_DQK];
        for (int c = 0; c < OR_DQK; ++c) qh[c] = oracle_bf16_to_f64(q[(r * H + h) * OR_DQK + c]);
        double* lg = (double*)malloc(sizeof(double) * (size_t)k);
        double m = -INFINITY;
        for (int j = 0; j < k; ++j) {
            if (sel[j] < 0) {
                lg[j] = -INFINITY;
                continue;
            }
            const uint16_t* row = kv + ((int64_t)off[b] + sel[j]) * OR_DQK;
            double dot = 0.0;
            for (int c = 0; c < OR_DQK; ++c) dot += qh[c] * oracle_bf16_to_f64(row[c]);
            macs += OR_DQK;
            lg[j] = dot * scale;
            if (lg[j] > m) m = lg[j];
        }
        double* o = out + (i * H + h) * OR_DV;
        for (int c = 0; c < OR_DV; ++c) o[c] = 0.0;
        if (m == -INFINITY) {
            if (lse) lse[i * H + h] = -INFINITY;
            free(lg);
            continue;
        }
        double denom = 0.0;
        for (int j = 0; j < k; ++j) {
            if (sel[j] < 0) continue;
            double p = exp(lg[j] - m);
            denom += p;
            const uint16_t* row = kv + ((int64_t)off[b] + sel[j]) * OR_DQK;
            for (int c = 0; c < OR_DV; ++c) o[c] += p * oracle_bf16_to_f64(row[c]);
            macs += OR_DV;
        }
        for (int c = 0; c < OR_DV; ++c) o[c] /= denom;
        if (lse) lse[i * H + h] = m + log(denom);
        free(lg);
    }
    if (mac_count) *mac_count = macs;
    return OR_OK;
}

/* ---- 4. dense causal MLA (no selection) -------------------------------- */
/*
 * The same absorbed attention over every causally valid position
 * (s < E and s <= start + t): what the decode listing computes before the
 * index mask is added.  Written as its own loop so that the invariant
 * "sparse == dense when end_pos <= topk" compares two independent codes.
 */
int oracle_dense_mla(const uint16_t* q, const uint16_t* kv, const int32_t* off, int B, int T,
                     int H, double scale, const int64_t* rows, int64_t n_rows, double* out,
                     double* lse, int64_t* mac_count) {
    if (!q || !kv || !out || H <= 0) return OR_EINVAL;
    if (!rows) n_rows = (int64_t)B * T;
    if (check_common(off, B, T, rows, n_rows)) return OR_EINVAL;
    int64_t macs = 0;
#pragma omp parallel for schedule(dynamic, 1) reduction(+ : macs)
    for (int64_t ih = 0; ih < n_rows * H; ++ih) {
        int64_t i = ih / H;
        int h = (int)(ih % H);
        int64_t r = rows ? rows[i] : i;
        int b, t;
        int64_t E, t_abs;
        row_geometry(off, T, r, &b, &t, &E, &t_abs);
        int64_t n = t_abs + 1 < E ? t_abs + 1 : E;
        double qh[OR_DQK];
        for (int c = 0; c < OR_DQK; ++c) qh[c] = oracle_bf16_to_f64(q[(r * H + h) * OR_DQK + c]);
        double* lg = (double*)malloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
        double m = -INFINITY;
        for (int64_t s = 0; s < n; ++s) {
            const uint16_t* row = kv + ((int64_t)off[b] + s) * OR_DQK;
            double dot = 0.0;
            for (int c = 0; c < OR_DQK; ++c) dot += qh[c] * oracle_bf16_to_f64(row[c]);
            macs += OR_DQK;
            lg[s] = dot * scale;
            if (lg[s] > m) m = lg[s];
        }
        double denom = 0.0;
        double* o = out + (i * H + h) * OR_DV;
        for (int c = 0; c < OR_DV; ++c) o[c] = 0.0;
        for (int64_t s = 0; s < n; ++s) {
            double p = exp(lg[s] - m);
            denom += p;
            const uint16_t* row = kv + ((int64_t)off[b] + s) * OR_DQK;
            for (int c = 0; c < OR_DV; ++c) o[c] += p * oracle_bf16_to_f64(row[c]);
            macs += OR_DV;
        }
        for (int c = 0; c < OR_DV; ++c) o[c] = n > 0 ? o[c] / denom : 0.0;
        if (lse) lse[i * H + h] = n > 0 ? m + log(denom) : -INFINITY;
        free(lg);
    }
    if (mac_count) *mac_count = macs;
    return OR_OK;
}

/* ---- 5. indexer pre-stage: rotary embedding, then rotate_activation ---- */
/*
 * [Sel] Indexer.forward, before act_quant: q (per head) and k are split into
 * the rope part (the first rope_head_dim = 64 entries) and the rest; the rope
 * part gets apply_rotary_emb(., freqs_cis, False) -- "rope in indexer is not
 * interleaved" -- the two parts are joined again, and the 128-vector goes
 * through rotate_activation.  Neither function is printed on the pages.
 * Readings taken:
 *   - not interleaved: rope entry i (i < 32) is paired with entry i + 32,
 *     and the pair (a, b) becomes (a*cos_i - b*sin_i, a*sin_i + b*cos_i),
 *     the rotation by the angle whose cos/sin are freqs_cis[pos][i]; the
 *     table is an input (the pages give no rope base);
 *   - rotate_activation: the Walsh-Hadamard transform of the 128 entries in
 *     Sylvester order, H[i][j] = (-1)^popcount(i & j), scaled by 128^-1/2 so
 *     that it is a rotation (the pages name
 *     fast_hadamard_transform.hadamard_transform, and a replacement of it by
 *     a plain linear layer);
 *   - precision (round_bf16 != 0): q and k are bf16 tensors in the model, so
 *     the rotated rope part and the transform's output are each rounded to
 *     the nearest bf16 (ties to even); everything else is exact.  With
 *     round_bf16 == 0 nothing is rounded.
 * The transform is the matrix product written out, not a butterfly.
 * Vector v belongs to row v / vec_per_row, whose position is pos[row].
 */
static double round_bf16_f64(double v) {
    if (v == 0.0 || !isfinite(v)) return v;
    int e;
    const double m = frexp(v, &e);             /* v = m * 2^e, 0.5 <= |m| < 1 */
    return ldexp(nearbyint(ldexp(m, 8)), e - 8); /* 8 significant bits, ties to even */
}

static int popcount_int(int x) {
    int c = 0;
    for (; x; x >>= 1) c += x & 1;
    return c;
}

int oracle_rope_hadamard(const uint16_t* x, int64_t n_rows, int vec_per_row, const int32_t* pos,
                         const float* rope_cos, const float* rope_sin, int64_t rope_len, int round_bf16,
                         double* y) {
    if (!x || !pos || !rope_cos || !rope_sin || !y || n_rows < 0 || vec_per_row <= 0 || rope_len <= 0)
        return OR_EINVAL;
    for (int64_t r = 0; r < n_rows; ++r)
        if (pos[r] < 0 || pos[r] >= rope_len) return OR_EINVAL;
    const double scale = 1.0 / sqrt((double)OR_DI);
#pragma omp parallel for schedule(static)
    for (int64_t v = 0; v < n_rows * vec_per_row; ++v) {
        const int64_t p = pos[v / vec_per_row];
        double a[OR_DI];
        for (int d = 0; d < OR_DI; ++d) a[d] = oracle_bf16_to_f64(x[v * OR_DI + d]);
        double u[OR_DI];
        for (int i = 0; i < 32; ++i) {
            const double c = rope_cos[p * 32 + i], sn = rope_sin[p * 32 + i];
            u[i] = a[i] * c - a[i + 32] * sn;
            u[i + 32] = a[i] * sn + a[i + 32] * c;
        }
        for (int d = 64; d < OR_DI; ++d) u[d] = a[d];
        if (round_bf16)
            for (int d = 0; d < 64; ++d) u[d] = round_bf16_f64(u[d]);
        for (int i = 0; i < OR_DI; ++i) {
            double acc = 0.0;
            for (int j = 0; j < OR_DI; ++j) acc += (popcount_int(i & j) & 1) ? -u[j] : u[j];
            acc *= scale;
            y[v * OR_DI + i] = round_bf16 ? round_bf16_f64(acc) : acc;
        }
    }
    return OR_OK;
}

int oracle_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}
