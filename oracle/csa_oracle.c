/*
 * CPU oracle for hybrid compressed attention (CSA / HCA).  TEST INFRASTRUCTURE ONLY:
 * used by tests/, the smoke check and the benchmark's CPU baseline leg; never by the
 * product path.  Plain loops, fp64 arithmetic, no blocking or fusion.  See csa_oracle.h
 * for the conventions and the page passages each step follows.
 *
 * Build: gcc -O2 -fopenmp -fPIC -shared -ffp-contract=off (no fast-math: the indexer score
 * is defined in fp32 with explicit fmaf and must not be re-associated).
 */
#include "csa_oracle.h"

#include <math.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

int orc_num_threads(void) {
#ifdef _OPENMP
    return omp_get_max_threads();
#else
    return 1;
#endif
}

/* ------------------------------------------------------------------------------------ */
/* Storage number formats.  BF16: 1 sign, 8 exponent (bias 127), 7 stored mantissa bits.
 * E4M3 "fn" (the FP8 format of the pages' 1x128 quantisation): 1 sign, 4 exponent
 * (bias 7), 3 mantissa bits, largest finite 448, no infinities, S.1111.111 is NaN.      */

double orc_bf16_value(uint16_t bits) {
    uint32_t u = (uint32_t)bits << 16;
    float f;
    memcpy(&f, &u, 4);
    return (double)f;
}

/* Round x to the nearest bf16 (ties to even).  The value grid in the binade
 * [2^(E-1), 2^E) has spacing 2^(E-8) (8 significant bits); below 2^-126 the spacing is
 * fixed at 2^-133 (subnormals).  rint() rounds half to even in the default mode. */
uint16_t orc_bf16_round(double x) {
    if (isnan(x)) return 0x7FC0;
    uint16_t sign = signbit(x) ? 0x8000 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    if (isinf(a)) return sign | 0x7F80;
    int E;
    frexp(a, &E);
    int qexp = E - 8;
    if (qexp < -133) qexp = -133;
    double v = ldexp(rint(ldexp(a, -qexp)), qexp);
    if (v >= 0x1.0p128) return sign | 0x7F80;
    float f = (float)v; /* exact: v lies on the bf16 grid */
    uint32_t u;
    memcpy(&u, &f, 4);
    return sign | (uint16_t)(u >> 16);
}

double orc_e4m3_value(uint8_t code) {
    int s = code >> 7, e = (code >> 3) & 0xF, mt = code & 7;
    if (e == 15 && mt == 7) return NAN;
    double v = (e == 0) ? ldexp((double)mt, -9) : ldexp((double)(8 + mt), e - 10);
    return s ? -v : v;
}

/* Round x to the nearest e4m3 value (ties to even), saturating to +-448.  Grid spacing is
 * 2^(E-4) in the binade [2^(E-1), 2^E) (4 significant bits) and 2^-9 below 2^-6. */
uint8_t orc_e4m3_round(double x) {
    if (isnan(x)) return 0x7F;
    uint8_t sign = signbit(x) ? 0x80 : 0;
    double a = fabs(x);
    if (a == 0.0) return sign;
    double v;
    if (isinf(a)) {
        v = 448.0;
    } else {
        int E;
        frexp(a, &E);
        int qexp = E - 4;
        if (qexp < -9) qexp = -9;
        v = ldexp(rint(ldexp(a, -qexp)), qexp);
        if (v > 448.0) v = 448.0;
    }
    if (v == 0.0) return sign;
    int E2;
    double f = frexp(v, &E2); /* v = f * 2^E2, f in [0.5, 1) -> v = (2f) * 2^(E2-1) */
    int be = E2 - 1 + 7;      /* biased exponent */
    uint8_t code;
    if (be >= 1) {
        int mt = (int)((2.0 * f - 1.0) * 8.0); /* exact: 3 fraction bits */
        code = (uint8_t)((be << 3) | mt);
    } else {
        code = (uint8_t)(int)ldexp(v, 9); /* subnormal: v = mt * 2^-9 */
    }
    return sign | code;
}

void orc_bf16_round_array(const double* x, int64_t n, uint16_t* out) {
    for (int64_t i = 0; i < n; i++) out[i] = orc_bf16_round(x[i]);
}

void orc_e4m3_round_array(const double* x, int64_t n, uint8_t* out) {
    for (int64_t i = 0; i < n; i++) out[i] = orc_e4m3_round(x[i]);
}

/* ------------------------------------------------------------------------------------ */
/* Partial RoPE ([P2] "其他注意力技术细节": rotary embedding on the last 64 dims of query and
 * KV only; [P4]: only the last 64 dimensions are rotated).  Interleaved pairs. */
void orc_rope(double* x, int D, double pos, double theta) {
    for (int j = 0; j < 32; j++) {
        double inv_freq = pow(theta, -(2.0 * j) / 64.0);
        double a = pos * inv_freq;
        double c = cos(a), s = sin(a);
        double* p = x + (D - 64) + 2 * j;
        double x0 = p[0], y0 = p[1];
        p[0] = x0 * c - y0 * s;
        p[1] = x0 * s + y0 * c;
    }
}

/* RMSNorm with unit weight over all D channels ([P2] QK-norm / [P4] "QK-norms"). */
void orc_rmsnorm(double* x, int D, double eps) {
    double ss = 0.0;
    for (int c = 0; c < D; c++) ss += x[c] * x[c];
    double r = 1.0 / sqrt(ss / D + eps);
    for (int c = 0; c < D; c++) x[c] *= r;
}

/* ------------------------------------------------------------------------------------ */
/* Entry storage ([P2] "混合精度存储": RoPE dims in BF16, the rest FP8; [P4]: FP8 scheme with
 * 1x128 blocks).  Format 1 row: 512 e4m3 codes | 4 fp32 scales | 64 bf16. */
int orc_entry_row_bytes(int fmt, int D) {
    if (fmt == 0) return 2 * D;
    if (fmt == 1 && D == 576) return 512 + 16 + 128;
    return -1;
}

void orc_entry_store(const double* e, int fmt, int D, uint8_t* row) {
    if (fmt == 0) {
        for (int c = 0; c < D; c++) {
            uint16_t b = orc_bf16_round(e[c]);
            memcpy(row + 2 * c, &b, 2);
        }
        return;
    }
    /* fmt 1, D = 576 */
    for (int blk = 0; blk < 4; blk++) {
        double amax = 0.0;
        for (int c = 128 * blk; c < 128 * blk + 128; c++) amax = fmax(amax, fabs(e[c]));
        float scale = (float)(amax / 448.0);
        if (!(scale > 0.0f)) scale = 1.0f;
        for (int c = 128 * blk; c < 128 * blk + 128; c++)
            row[c] = orc_e4m3_round(e[c] / (double)scale);
        memcpy(row + 512 + 4 * blk, &scale, 4);
    }
    for (int c = 512; c < 576; c++) {
        uint16_t b = orc_bf16_round(e[c]);
        memcpy(row + 528 + 2 * (c - 512), &b, 2);
    }
}

void orc_entry_load(const uint8_t* row, int fmt, int D, double* e) {
    if (fmt == 0) {
        for (int c = 0; c < D; c++) {
            uint16_t b;
            memcpy(&b, row + 2 * c, 2);
            e[c] = orc_bf16_value(b);
        }
        return;
    }
    for (int blk = 0; blk < 4; blk++) {
        float scale;
        memcpy(&scale, row + 512 + 4 * blk, 4);
        for (int c = 128 * blk; c < 128 * blk + 128; c++)
            e[c] = orc_e4m3_value(row[c]) * (double)scale;
    }
    for (int c = 512; c < 576; c++) {
        uint16_t b;
        memcpy(&b, row + 528 + 2 * (c - 512), 2);
        e[c] = orc_bf16_value(b);
    }
}

/* ------------------------------------------------------------------------------------ */
/* Steps a1/a2: compression of one entry.
 * [P2] 2.1 CSA: every m=4 tokens become one entry; each entry draws on 2m=8 tokens
 * (current block and the previous one).  [P2] 2.1 HCA: every m'=128 tokens, one block.
 * Pooling per channel c: weights = softmax over the pooled tokens of (gate + bias row j),
 * entry = weighted sum of the raw KV; then RMSNorm; then RoPE at the block-end position. */
static int compress_one(const uint16_t* kv, const uint16_t* gate, const float* bias,
                        int64_t row0, int64_t pos0, int64_t i, int m, int span, int D,
                        double theta, double eps, double* e) {
    int64_t first = (i + 1) * (int64_t)m - span;
    for (int j = 0; j < span; j++) {
        int64_t p = first + j;
        if (p >= 0 && p < pos0) return -1; /* needed raw token not stored */
    }
    for (int c = 0; c < D; c++) {
        double mx = -INFINITY;
        for (int j = 0; j < span; j++) {
            int64_t p = first + j;
            if (p < 0) continue; /* first CSA entry: no previous block */
            double l = orc_bf16_value(gate[(row0 + p - pos0) * D + c]) + (double)bias[j * D + c];
            if (l > mx) mx = l;
        }
        double den = 0.0, num = 0.0;
        for (int j = 0; j < span; j++) {
            int64_t p = first + j;
            if (p < 0) continue;
            int64_t r = row0 + p - pos0;
            double l = orc_bf16_value(gate[r * D + c]) + (double)bias[j * D + c];
            double wgt = exp(l - mx);
            den += wgt;
            num += wgt * orc_bf16_value(kv[r * D + c]);
        }
        e[c] = num / den;
    }
    orc_rmsnorm(e, D, eps);
    orc_rope(e, D, (double)((i + 1) * (int64_t)m - 1), theta);
    return 0;
}

int orc_compress(const uint16_t* kv, const uint16_t* gate, const float* bias,
                 const int64_t* kv_off, const int64_t* kv_pos0, const int64_t* ent_off,
                 const int32_t* item_seq, const int32_t* item_ent, int64_t n_items,
                 int m, int span, int D, int fmt, double theta, double eps,
                 uint8_t* entries, double* e_f64) {
    int rc = 0;
    int row_bytes = orc_entry_row_bytes(fmt, D);
    if (row_bytes < 0) return -4;
#pragma omp parallel for schedule(dynamic, 16)
    for (int64_t n = 0; n < n_items; n++) {
        int b = item_seq[n];
        int64_t i = item_ent[n];
        double* e = (double*)malloc(sizeof(double) * D);
        int r = compress_one(kv, gate, bias, kv_off[b], kv_pos0[b], i, m, span, D, theta, eps, e);
        if (r != 0) {
#pragma omp atomic write
            rc = r;
        } else {
            if (entries) orc_entry_store(e, fmt, D, entries + (ent_off[b] + i) * row_bytes);
            if (e_f64) memcpy(e_f64 + n * D, e, sizeof(double) * D);
        }
        free(e);
    }
    return rc;
}

/* ------------------------------------------------------------------------------------ */
/* Steps a3/a4: lightning indexer and top-k ([P2] 2.1 CSA "稀疏选择": the lightning indexer
 * picks the top-k compressed entries; k = 1024 (Pro) or 512 (Flash)). */

typedef struct {
    float s;
    int32_t i;
} scored_t;

/* Total order of the selection: larger score first, lower index first among equal scores
 * (float comparison treats -0 and +0 as equal). */
static int by_score_desc(const void* a, const void* b) {
    const scored_t* x = (const scored_t*)a;
    const scored_t* y = (const scored_t*)b;
    if (x->s > y->s) return -1;
    if (x->s < y->s) return 1;
    return (x->i < y->i) ? -1 : (x->i > y->i);
}

static int by_index(const void* a, const void* b) {
    int32_t x = *(const int32_t*)a, y = *(const int32_t*)b;
    return (x < y) ? -1 : (x > y);
}

static void select_topk(const float* s, int n, int k, int32_t* out) {
    scored_t* all = (scored_t*)malloc(sizeof(scored_t) * (n > 0 ? n : 1));
    for (int i = 0; i < n; i++) {
        all[i].s = s[i];
        all[i].i = i;
    }
    qsort(all, (size_t)n, sizeof(scored_t), by_score_desc);
    int take = n < k ? n : k;
    for (int j = 0; j < take; j++) out[j] = all[j].i;
    qsort(out, (size_t)take, sizeof(int32_t), by_index);
    for (int j = take; j < k; j++) out[j] = -1;
    free(all);
}

int orc_indexer_topk(const uint8_t* qI, const float* qs, const float* w,
                     const uint8_t* kI, const float* ks, const int64_t* ent_off,
                     const int32_t* q_seq, const int32_t* q_pos, int Q, int HI, int dI,
                     int m, int k, int32_t* idx_out, float* scores, int64_t ld_scores) {
    int rc = 0;
#pragma omp parallel for schedule(dynamic, 1)
    for (int qq = 0; qq < Q; qq++) {
        int b = q_seq[qq];
        int64_t t = q_pos[qq];
        int n = (int)((t + 1) / m);
        if (scores && n > ld_scores) {
#pragma omp atomic write
            rc = -3;
            continue;
        }
        float* ws = (float*)malloc(sizeof(float) * HI);
        double* qv = (double*)malloc(sizeof(double) * HI * dI);
        double* kvv = (double*)malloc(sizeof(double) * dI);
        float* s = (float*)malloc(sizeof(float) * (n > 0 ? n : 1));
        for (int h = 0; h < HI; h++) ws[h] = w[(int64_t)qq * HI + h] * qs[(int64_t)qq * HI + h];
        for (int x = 0; x < HI * dI; x++) qv[x] = orc_e4m3_value(qI[(int64_t)qq * HI * dI + x]);
        int bad = 0;
        for (int i = 0; i < n; i++) {
            int64_t row = ent_off[b] + i;
            for (int c = 0; c < dI; c++) kvv[c] = orc_e4m3_value(kI[row * dI + c]);
            float acc = 0.0f;
            for (int h = 0; h < HI; h++) {
                double dot = 0.0; /* exact: e4m3 products have <= 8 significant bits */
                for (int c = 0; c < dI; c++) dot += qv[h * dI + c] * kvv[c];
                float d = (float)dot;
                acc = fmaf(ws[h], fmaxf(d, 0.0f), acc);
            }
            s[i] = acc * ks[row];
            if (isnan(s[i])) bad = 1;
        }
        if (bad) {
#pragma omp atomic write
            rc = -2;
        }
        select_topk(s, n, k, idx_out + (int64_t)qq * k);
        if (scores) memcpy(scores + (int64_t)qq * ld_scores, s, sizeof(float) * n);
        free(ws);
        free(qv);
        free(kvv);
        free(s);
    }
    return rc;
}

/* ------------------------------------------------------------------------------------ */
/* Steps a3/a4 in FP4 ([P2] Figure 2 "Lightning Indexer FP4 Precision"; section 3.4: MXFP4
 * on the QK path of CSA, indexer scores quantised FP32 -> BF16 for the top-k selector).  */

/* FP4 E2M1: sign bit 3, exponent bits 2..1 (bias 1), mantissa bit 0.  Exponent field 0 is
 * subnormal: 0.5 * mantissa. */
double orc_e2m1_value(uint8_t code) {
    int sign = (code >> 3) & 1, e = (code >> 1) & 3, mant = code & 1;
    double v = (e == 0) ? 0.5 * mant : ldexp(1.0 + 0.5 * mant, e - 1);
    return sign ? -v : v;
}

/* E8M0: an unsigned biased exponent, 2^(e-127); all ones is NaN. */
double orc_e8m0_value(uint8_t code) {
    if (code == 0xFF) return NAN;
    return ldexp(1.0, (int)code - 127);
}

/* Element c of a packed MXFP4 vector. */
static double mxfp4_elem(const uint8_t* packed, int c) {
    uint8_t byte = packed[c >> 1];
    return orc_e2m1_value((c & 1) ? (uint8_t)(byte >> 4) : (uint8_t)(byte & 0x0F));
}

int orc_indexer_topk_mxfp4(const uint8_t* qI, const uint8_t* qI_sf, const float* w,
                           const uint8_t* kI, const uint8_t* kI_sf, const int64_t* ent_off,
                           const int32_t* q_seq, const int32_t* q_pos, int Q, int HI, int dI,
                           int m, int k, int select_bf16, int32_t* idx_out, float* scores,
                           int64_t ld_scores) {
    int rc = 0;
    const int nb = dI / 32;
#pragma omp parallel for schedule(dynamic, 1)
    for (int qq = 0; qq < Q; qq++) {
        int b = q_seq[qq];
        int64_t t = q_pos[qq];
        int n = (int)((t + 1) / m);
        if (scores && n > ld_scores) {
#pragma omp atomic write
            rc = -3;
            continue;
        }
        double* qv = (double*)malloc(sizeof(double) * HI * dI);
        double* qsc = (double*)malloc(sizeof(double) * HI * nb);
        double* kvv = (double*)malloc(sizeof(double) * dI);
        double* ksc = (double*)malloc(sizeof(double) * nb);
        float* s = (float*)malloc(sizeof(float) * (n > 0 ? n : 1));
        for (int h = 0; h < HI; h++) {
            const uint8_t* qp = qI + ((int64_t)qq * HI + h) * (dI / 2);
            for (int c = 0; c < dI; c++) qv[h * dI + c] = mxfp4_elem(qp, c);
            for (int bl = 0; bl < nb; bl++)
                qsc[h * nb + bl] = orc_e8m0_value(qI_sf[((int64_t)qq * HI + h) * nb + bl]);
        }
        int bad = 0;
        for (int i = 0; i < n; i++) {
            int64_t row = ent_off[b] + i;
            for (int c = 0; c < dI; c++) kvv[c] = mxfp4_elem(kI + row * (dI / 2), c);
            for (int bl = 0; bl < nb; bl++) ksc[bl] = orc_e8m0_value(kI_sf[row * nb + bl]);
            float acc = 0.0f;
            for (int h = 0; h < HI; h++) {
                double dot = 0.0;
                for (int bl = 0; bl < nb; bl++) {
                    double blk = 0.0; /* exact: products of E2M1 values have <= 4 bits */
                    for (int c = 32 * bl; c < 32 * bl + 32; c++) blk += qv[h * dI + c] * kvv[c];
                    dot += blk * qsc[h * nb + bl] * ksc[bl];
                }
                float d = (float)dot;
                acc = fmaf(w[(int64_t)qq * HI + h], fmaxf(d, 0.0f), acc);
            }
            if (select_bf16) acc = (float)orc_bf16_value(orc_bf16_round((double)acc));
            s[i] = acc;
            if (isnan(s[i])) bad = 1;
        }
        if (bad) {
#pragma omp atomic write
            rc = -2;
        }
        select_topk(s, n, k, idx_out + (int64_t)qq * k);
        if (scores) memcpy(scores + (int64_t)qq * ld_scores, s, sizeof(float) * n);
        free(qv);
        free(qsc);
        free(kvv);
        free(ksc);
        free(s);
    }
    return rc;
}

/* ------------------------------------------------------------------------------------ */
/* Steps a5/a6: shared-KV MQA over compressed entries plus the sliding window, with an
 * attention sink and partial / inverse RoPE.
 * [P2] 2.1: CSA attends to the top-k entries, HCA densely to all entries; both add a
 * 128-token sliding-window branch.  [P2] "Shared Key-Value MQA": each entry is both key
 * and value.  "Attention Sink": learnable sink logits, weights may sum to less than 1.
 * "Partial RoPE": RoPE on the last 64 dims of q and KV, inverse RoPE on the output.
 * Output for head h:  o = sum_j e^(l_j - M) v_j / (e^(sink - M) + sum_j e^(l_j - M)),
 * l_j = scale * <RoPE_t(q_h), k_j>, M = max(sink, max_j l_j), then o <- RoPE_{-t}(o). */
int orc_attention(const uint16_t* q, const uint8_t* entries, int fmt, const int64_t* ent_off,
                  const uint16_t* kv, const int64_t* kv_off, const int64_t* kv_pos0,
                  const int32_t* q_seq, const int32_t* q_pos, const int32_t* idx, int k,
                  int m, const float* sink, int Q, int H, int D, int W,
                  double scale, double theta, double eps, double* out) {
    int rc = 0;
    int row_bytes = orc_entry_row_bytes(fmt, D);
    if (row_bytes < 0) return -4;
#pragma omp parallel for schedule(dynamic, 1)
    for (int qq = 0; qq < Q; qq++) {
        int b = q_seq[qq];
        int64_t t = q_pos[qq];
        int64_t n = (t + 1) / m;
        int64_t w0 = t - W + 1 > 0 ? t - W + 1 : 0;
        int64_t n_win = W > 0 ? t - w0 + 1 : 0;
        int64_t n_ent = idx ? k : n;
        double* keys = (double*)malloc(sizeof(double) * (size_t)(n_ent + n_win) * D);
        int64_t nk = 0;
        int bad = 0;
        for (int64_t j = 0; j < n_ent; j++) {
            int64_t e = idx ? idx[(int64_t)qq * k + j] : j;
            if (e < 0) continue; /* padding */
            if (e >= n) {
                bad = 1;
                continue;
            }
            orc_entry_load(entries + (ent_off[b] + e) * row_bytes, fmt, D, keys + nk * D);
            nk++;
        }
        for (int64_t p = w0; p < w0 + n_win; p++) {
            if (p < kv_pos0[b]) {
                bad = 1;
                continue;
            }
            const uint16_t* raw = kv + (kv_off[b] + p - kv_pos0[b]) * D;
            double* r = keys + nk * D;
            for (int c = 0; c < D; c++) r[c] = orc_bf16_value(raw[c]);
            orc_rmsnorm(r, D, eps);
            orc_rope(r, D, (double)p, theta);
            nk++;
        }
        double* qh = (double*)malloc(sizeof(double) * D);
        double* lg = (double*)malloc(sizeof(double) * (nk > 0 ? nk : 1));
        for (int h = 0; h < H; h++) {
            const uint16_t* qraw = q + ((int64_t)qq * H + h) * D;
            for (int c = 0; c < D; c++) qh[c] = orc_bf16_value(qraw[c]);
            orc_rope(qh, D, (double)t, theta);
            double M = (double)sink[h];
            for (int64_t j = 0; j < nk; j++) {
                double dot = 0.0;
                for (int c = 0; c < D; c++) dot += qh[c] * keys[j * D + c];
                lg[j] = scale * dot;
                if (lg[j] > M) M = lg[j];
            }
            double den = exp((double)sink[h] - M);
            double* o = out + ((int64_t)qq * H + h) * D;
            for (int c = 0; c < D; c++) o[c] = 0.0;
            for (int64_t j = 0; j < nk; j++) {
                double p = exp(lg[j] - M);
                den += p;
                for (int c = 0; c < D; c++) o[c] += p * keys[j * D + c];
            }
            for (int c = 0; c < D; c++) o[c] /= den;
            orc_rope(o, D, -(double)t, theta);
        }
        if (bad) {
#pragma omp atomic write
            rc = -1;
        }
        free(qh);
        free(lg);
        free(keys);
    }
    return rc;
}
