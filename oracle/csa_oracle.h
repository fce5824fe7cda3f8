/*
 * CPU oracle for hybrid compressed attention (CSA / HCA).
 *
 * TEST INFRASTRUCTURE ONLY.  This is a plain, slow, fp64 restatement of what the
 * method computes, used by the test-suite, the smoke check and the CPU baseline leg of
 * the benchmark to judge the CUDA library.  Product code must never link, load or call
 * it, and it shares no code, header, table or helper with the CUDA library.
 *
 * Sources (web pages on the DeepSeek-V4 technical report):
 *   [P2] "DeepSeek-V4 深度分析报告" (juejin.cn), section 2.1 "混合注意力架构：CSA + HCA"
 *        (CSA: 4:1 overlapped compression, lightning indexer, top-k, 128-token window;
 *         HCA: 128:1 single-block compression, dense attention; Figure 2),
 *        "其他注意力技术细节" (shared-KV MQA, partial RoPE on the last 64 dims with inverse
 *         RoPE on the output, learnable attention sink, BF16 RoPE dims / FP8 others),
 *        section 3.3 (batch invariance), section 3.5 (state cache / classical cache).
 *   [P4] stuffyNLP post 255 on DeepSeek-V4 (ml-brand.github.io): CSA stride m, 2m tokens
 *        per entry, m=4; HCA m'=128; partial RoPE on the last 64 dims; FP8 1x128 blocks.
 * Where the pages leave a step open, the problem statement of this library fixes it:
 * per-channel softmax pooling of gate logits + learned positional bias, RMSNorm, RoPE on
 * the last 64 dims at the block-end position; indexer score sum_h w_h * ReLU(q_h . k).
 *
 * Parity status: every function below is pinned by the CPU tests in tests/test_oracle_*.py
 * (closed forms, limits, library special cases, brute force).  None is "parity unpinned".
 *
 * Conventions (readings of the pages, listed with reasons in the design notes):
 *   - bf16 / e4m3 values are passed as raw storage bits (uint16_t / uint8_t).
 *   - RoPE: interleaved pairs (D-64+2j, D-64+2j+1), j=0..31, inv_freq_j = theta^(-2j/64),
 *     (x, y) -> (x cos a - y sin a, x sin a + y cos a), a = pos * inv_freq_j.
 *   - Compressed entry i pools positions (i+1)*m - span .. (i+1)*m - 1 (span = 2m for CSA,
 *     m for HCA); positions < 0 are dropped; bias row j goes with the j-th pooled position;
 *     RoPE at the block-end position (i+1)*m - 1.
 *   - Entry i is visible to a query at position t iff (i+1)*m - 1 <= t.
 *   - Window: raw tokens max(0, t-W+1) .. t, each RMSNormed and RoPEd at its own position.
 *   - Entry storage formats: 0 = D bf16 values; 1 = D=576 row of 656 bytes:
 *     512 e4m3 codes (channels 0..511), 4 fp32 scales (one per 128 channels, value =
 *     code * scale), 64 bf16 values (channels 512..575).
 */
#ifndef CSA_ORACLE_H
#define CSA_ORACLE_H
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* ---- storage number formats ---- */
double orc_bf16_value(uint16_t bits);
uint16_t orc_bf16_round(double x);          /* round-to-nearest-even, overflow -> inf */
double orc_e4m3_value(uint8_t code);        /* e4m3 "fn": no inf, 0x7f/0xff are NaN */
uint8_t orc_e4m3_round(double x);           /* round-to-nearest-even, saturate to +-448 */
void orc_bf16_round_array(const double* x, int64_t n, uint16_t* out);
void orc_e4m3_round_array(const double* x, int64_t n, uint8_t* out);

/* ---- building blocks ---- */
void orc_rope(double* x, int D, double pos, double theta);   /* in place, last 64 dims */
void orc_rmsnorm(double* x, int D, double eps);              /* in place, weight 1 */
int orc_entry_row_bytes(int fmt, int D);
void orc_entry_store(const double* e, int fmt, int D, uint8_t* row);
void orc_entry_load(const uint8_t* row, int fmt, int D, double* e);

/* ---- step a1/a2: compression ----
 * Computes compressed entries item_ent[n] of sequences item_seq[n].
 * kv, gate: bf16 rows [*, D]; position p of sequence b is row kv_off[b] + p - kv_pos0[b].
 * bias: fp32 [span, D].  Writes stored rows to entries (row ent_off[b] + i, fmt) when
 * entries != NULL and the fp64 values before storage rounding to e_f64 [n_items, D] when
 * e_f64 != NULL.  Returns 0, or -1 when a needed position is not stored. */
int orc_compress(const uint16_t* kv, const uint16_t* gate, const float* bias,
                 const int64_t* kv_off, const int64_t* kv_pos0, const int64_t* ent_off,
                 const int32_t* item_seq, const int32_t* item_ent, int64_t n_items,
                 int m, int span, int D, int fmt, double theta, double eps,
                 uint8_t* entries, double* e_f64);

/* ---- steps a3/a4: lightning indexer score + top-k ----
 * qI e4m3 [Q, HI, dI], qs fp32 [Q, HI], w fp32 [Q, HI]; kI e4m3 [rows, dI], ks fp32 [rows];
 * entry i of sequence b is row ent_off[b] + i.  Visible entries n = floor((t+1)/m).
 * Score (fp32, fixed order): acc = +0; for h: acc = fmaf(w*qs, max(dot_h, 0), acc);
 * s = acc * ks, where dot_h is the exact dot product rounded once to fp32.
 * Top-k: order (score desc, index asc); emit ascending index; pad with -1.
 * scores (nullable): fp32 [Q, ld_scores], entries >= n left untouched.
 * Returns 0, or -2 on a NaN score, -3 when n > ld_scores for a non-null scores buffer. */
int orc_indexer_topk(const uint8_t* qI, const float* qs, const float* w,
                     const uint8_t* kI, const float* ks, const int64_t* ent_off,
                     const int32_t* q_seq, const int32_t* q_pos, int Q, int HI, int dI,
                     int m, int k, int32_t* idx_out, float* scores, int64_t ld_scores);

/* ---- steps a3/a4 in FP4: MXFP4 lightning indexer, FP32 or BF16 selector scores ----
 * [P2] Figure 2 ("Lightning Indexer FP4 Precision") and "其他注意力技术细节" (the indexer
 * computes in FP4); section 3.4 (MXFP4 quantisation on the QK path of CSA; the indexer
 * scores quantised from FP32 to BF16 for the top-k selector).
 * MXFP4 is the OCP microscaling format: FP4 E2M1 elements (1 sign, 2 exponent bits with
 * bias 1, 1 mantissa bit: +-{0, 0.5, 1, 1.5, 2, 3, 4, 6}) sharing one E8M0 scale per 32
 * consecutive elements (value 2^(e-127); e = 255 is NaN).  Storage: two elements per byte,
 * element 2j in the low nibble.
 * qI [Q, HI, dI/2] packed, qI_sf [Q, HI, dI/32]; w fp32 [Q, HI]; kI [rows, dI/2] packed,
 * kI_sf [rows, dI/32]; dI a multiple of 32.  The block scales carry the magnitudes, so
 * there is no per-head or per-entry factor besides w.
 * Score (fp32, fixed order): acc = +0; for h: acc = fmaf(w, max(dot_h, 0), acc); s = acc,
 * where dot_h = sum over blocks of 2^(eq + ek - 254) * (exact block dot of the elements),
 * summed in fp64 and rounded once to fp32.
 * select_bf16 = 0: top-k of s as in orc_indexer_topk.  select_bf16 = 1: each score is
 * rounded to BF16 (nearest, ties to even) first; the top-k is taken on the rounded values
 * with the same order (ties: lower index first), and scores receives the rounded values.
 * Returns as orc_indexer_topk. */
double orc_e2m1_value(uint8_t code);        /* the low 4 bits of code */
double orc_e8m0_value(uint8_t code);
int orc_indexer_topk_mxfp4(const uint8_t* qI, const uint8_t* qI_sf, const float* w,
                           const uint8_t* kI, const uint8_t* kI_sf, const int64_t* ent_off,
                           const int32_t* q_seq, const int32_t* q_pos, int Q, int HI, int dI,
                           int m, int k, int select_bf16, int32_t* idx_out, float* scores,
                           int64_t ld_scores);

/* ---- steps a5/a6: sparse (idx != NULL) or dense (idx == NULL) shared-KV MQA ----
 * q bf16 [Q, H, D]; entries in format fmt at rows ent_off[b] + i; kv raw bf16 window rows
 * addressed as in orc_compress.  n = floor((t+1)/m) entries are visible to a query at t.
 * Sparse: keys = entries idx[q, 0..k-1] that are >= 0 (each must be < n).
 * Dense: keys = entries 0 .. n-1.  Both add the window (W raw tokens ending at t).
 * sink fp32 [H].  out fp64 [Q, H, D].
 * Returns 0, or -1 when an index or a position is out of range. */
int orc_attention(const uint16_t* q, const uint8_t* entries, int fmt, const int64_t* ent_off,
                  const uint16_t* kv, const int64_t* kv_off, const int64_t* kv_pos0,
                  const int32_t* q_seq, const int32_t* q_pos, const int32_t* idx, int k,
                  int m, const float* sink, int Q, int H, int D, int W,
                  double scale, double theta, double eps, double* out);

int orc_num_threads(void);

#ifdef __cplusplus
}
#endif
#endif
