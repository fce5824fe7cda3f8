/*
 * libcsa -- hybrid compressed attention (CSA / HCA) for NVIDIA B200 (sm_100a).
 *
 * The method is described on the pages about the DeepSeek-V4 technical report:
 *   "DeepSeek-V4 深度分析报告" (juejin.cn), section 2.1 "混合注意力架构：CSA + HCA", its
 *   Figure 2, the list "其他注意力技术细节", section 3.3 (batch-invariant kernels) and
 *   section 3.5 (state cache / classical KV cache); and the stuffyNLP post 255 on
 *   DeepSeek-V4 (CSA stride m=4 with 2m tokens per entry, HCA m'=128, partial RoPE on the
 *   last 64 dims, FP8 with 1x128 blocks).
 *
 * Conventions shared by every call
 * --------------------------------
 *  - All tensor arguments are DEVICE pointers owned by the caller.  The library never
 *    allocates, frees or synchronises; each call only enqueues kernels on `stream`
 *    (a cudaStream_t passed as void*, NULL = legacy default stream) and returns.
 *  - Host-side validation happens before any launch.  On failure nothing is launched and
 *    the call returns a non-zero csa_status_t; csa_last_error() (thread-local) describes it.
 *  - `dev_status` (nullable device int32) collects CSA_DEV_* bits with atomicOr when a
 *    kernel meets data it must not use (an index outside the visible entries, a position
 *    that is not stored, a NaN score, too small a workspace).  The offending access is
 *    skipped; kernels never trap.  Read it after your own synchronisation.
 *  - bf16 tensors are passed as raw 16-bit storage, e4m3 as raw bytes ("fn" encoding,
 *    largest finite 448).  Row-major layouts throughout.
 *  - Ragged batches.  B sequences; seq_len[b] (int64) is the number of tokens sequence b
 *    holds so far (positions 0 .. seq_len[b]-1).  Raw per-token data (kv, gate) is a row
 *    store: position p of sequence b is row kv_off[b] + (p - kv_pos0[b]); only positions
 *    kv_pos0[b] .. seq_len[b]-1 are stored (a decode state cache keeps just the tail).
 *    Compressed entries and indexer keys share one entry numbering: entry i of sequence b
 *    is row ent_off[b] + i, for i < floor(seq_len[b]/m).  seq_len, kv_off, kv_pos0 and
 *    ent_off are int64 [B]; kernels check every position and index against them.
 *  - Queries: q_seq[Q] (int32, sequence) and q_pos[Q] (int32, token position
 *    0 <= t < seq_len[q_seq]; other queries set CSA_DEV_OOB and are skipped).  Entry i is
 *    visible to a query at t iff its block has ended: (i+1)*m - 1 <= t, so
 *    n_vis(t) = floor((t+1)/m).  The window is raw tokens max(0, t-W+1) .. t.
 *  - RoPE: interleaved pairs (D-64+2j, D-64+2j+1), j = 0..31, angle pos*theta^(-2j/64),
 *    (x, y) -> (x cos a - y sin a, x sin a + y cos a).  Angles are formed in fp64.
 *  - Batch invariance (section 3.3): every output element of a query is computed by the
 *    same instructions in the same order whatever the batch, the neighbours or the slot;
 *    no reduction of one query is split by batch size or SM count.
 */
#ifndef CSA_H
#define CSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    CSA_OK = 0,
    CSA_ERR_INVALID_ARG = 1,   /* null / misaligned pointer, bad size or enum */
    CSA_ERR_UNSUPPORTED = 2,   /* valid but not implemented shape (head dims, heads, k) */
    CSA_ERR_CUDA = 3,          /* a CUDA runtime call or a launch failed */
    CSA_ERR_WORKSPACE = 4      /* workspace missing or smaller than the query says */
} csa_status_t;

/* Bits OR-ed into *dev_status by kernels. */
#define CSA_DEV_OOB 1       /* index / position outside the visible or stored range (skipped) */
#define CSA_DEV_TIMEOUT 2   /* a bounded wait on a barrier gave up; the kernel returned */
#define CSA_DEV_NAN 4       /* a NaN indexer score */
#define CSA_DEV_CAPACITY 8  /* n_vis larger than the max_n the workspace was sized for */

/* Entry storage formats.
 * CSA_KV_BF16: D bf16 values per entry (row of 2*D bytes).
 * CSA_KV_FP8_576: D = 576 only; row of 656 bytes = 512 e4m3 codes for channels 0..511,
 *   4 fp32 scales at byte 512 (channel c of block c/128 has value code*scale; the scale is
 *   the block's absmax / 448), then 64 bf16 values for the RoPE channels 512..575
 *   ("混合精度存储": RoPE dims in BF16, the rest FP8; stuffyNLP: FP8 1x128 blocks). */
#define CSA_KV_BF16 0
#define CSA_KV_FP8_576 1

/*
 * Cache layout ("DeepSeek-V4 深度分析报告" 3.5, KV cache management: a fixed-size state
 * cache holds the sliding-window KV and the not yet compressed tail; the classical cache
 * holds the compressed CSA / HCA entries in blocks of lcm(m, m') = 128 tokens).  Passed by
 * pointer to the calls below; NULL keeps the contiguous layout described above.
 *   block_table  nullable int32 [B, bt_stride]: the classical cache in blocks of 128 tokens,
 *                i.e. 32 CSA entries (m = 4 only).  Entry i of sequence b is row
 *                block_table[b * bt_stride + i / 32] * 32 + i % 32 of the entry (and
 *                indexer-key) store; ent_off is then unused (may be NULL).  A block index
 *                < 0, or whose rows lie past ent_rows, sets CSA_DEV_OOB and its entries are
 *                skipped.  Dense HCA attention takes no block table (CSA_ERR_UNSUPPORTED).
 *   kv_ring      0: the raw store is linear as above.  > 0: the state cache is a ring of
 *                kv_ring rows per sequence; raw token p of sequence b is row
 *                kv_off[b] + p mod kv_ring, and positions seq_len[b] - kv_ring ..
 *                seq_len[b] - 1 are held (kv_pos0 is unused and may be NULL).  The ring
 *                must hold the window and the tokens an entry pools, else CSA_DEV_OOB.
 */
typedef struct {
    const int32_t* block_table;
    int64_t bt_stride;
    int64_t kv_ring;
} csa_cache_layout_t;

int csa_version(void);
const char* csa_last_error(void);
/* Bytes per stored entry row for (fmt, D), or -1 if unsupported. */
int32_t csa_entry_row_bytes(int32_t fmt, int32_t D);

/*
 * csa_compress -- CSA 4:1 overlapped KV compression (step a1).
 *   "DeepSeek-V4 深度分析报告" 2.1 CSA / Figure 2 "KV Compress 4:1 Overlapped": every
 *   m=4 tokens make one entry, and each entry pools 2m=8 tokens (its own block and the
 *   previous one).  For entry i: positions P = (i-1)*4 .. (i+1)*4-1 (positions < 0 are
 *   dropped, so entry 0 pools tokens 0..3 with bias rows 4..7); per channel c,
 *   w_j = softmax_j(gate[p_j, c] + pos_bias[j, c]), e_c = sum_j w_j * kv[p_j, c];
 *   then RMSNorm over all D channels (unit weight, epsilon eps); then RoPE on the last 64
 *   channels at the block-end position (i+1)*4 - 1; then stored in format fmt.
 * Arguments:
 *   kv, gate   bf16 [rows, D] raw KV and gate logits (row addressing as above)
 *   pos_bias   fp32 [8, D], row j pairs with the j-th pooled position
 *   item_seq, item_ent  int32 [n_items]: compute entry item_ent[n] of sequence item_seq[n]
 *   entries    output rows, format fmt; only the listed rows are written (with a block
 *              table in the layout, entry i's row comes from it; the caller provides rows
 *              for every block it names)
 *   layout     nullable cache layout (block table, state-cache ring)
 *   B          number of sequences (item_seq must be < B; the entry's last pooled
 *              position (i+1)*4-1 must be < seq_len[b], else CSA_DEV_OOB and no write)
 *   D          128 (fmt CSA_KV_BF16) or 576 (either format)
 * Pointers kv/gate/entries must be 16-byte aligned.  n_items = 0 is a no-op.
 * Errors: CSA_ERR_INVALID_ARG, CSA_ERR_UNSUPPORTED, CSA_ERR_CUDA; an entry whose tokens are
 * not stored sets CSA_DEV_OOB and is left unwritten.
 */
csa_status_t csa_compress(const void* kv, const void* gate, const float* pos_bias,
                          const int64_t* seq_len, const int64_t* kv_off, const int64_t* kv_pos0,
                          const int64_t* ent_off,
                          const int32_t* item_seq, const int32_t* item_ent, int64_t n_items,
                          int32_t B, int32_t D, int32_t fmt, float rope_theta, float eps,
                          void* entries, const csa_cache_layout_t* layout, int32_t* dev_status,
                          void* stream);

/*
 * hca_compress -- HCA 128:1 compression (step a2).
 *   "DeepSeek-V4 深度分析报告" 2.1 HCA / Figure 2 "KV Compress 128:1 Single Block": every
 *   m'=128 tokens make one entry, no overlap.  Entry i pools positions 128i .. 128i+127
 *   with the same per-channel softmax pooling, RMSNorm, and RoPE at position 128i+127.
 *   pos_bias is fp32 [128, D].  Other arguments as csa_compress.
 */
csa_status_t hca_compress(const void* kv, const void* gate, const float* pos_bias,
                          const int64_t* seq_len, const int64_t* kv_off, const int64_t* kv_pos0,
                          const int64_t* ent_off,
                          const int32_t* item_seq, const int32_t* item_ent, int64_t n_items,
                          int32_t B, int32_t D, int32_t fmt, float rope_theta, float eps,
                          void* entries, const csa_cache_layout_t* layout, int32_t* dev_status,
                          void* stream);

/*
 * lightning_indexer_topk -- lightning-indexer scores and top-k selection (steps a3, a4).
 *   "DeepSeek-V4 深度分析报告" 2.1 CSA "稀疏选择": a lightning indexer scores the compressed
 *   entries and keeps the top-k (k = 1024 for V4-Pro, 512 for V4-Flash); Figure 2.
 * For query q at t and every visible entry i < n_vis(t) of its sequence:
 *   d_h = sum_c qI[q,h,c] * kI[i,c]          (e4m3 products, fp32 accumulation)
 *   acc = +0; for h = 0..H_I-1: acc = fmaf(w[q,h] * qI_scale[q,h], max(d_h, 0), acc)
 *   s_i = acc * kI_scale[i]                  (all fp32, in this order)
 * idx_out[q, :] holds the k entries with the largest s_i (ties: lower i first), in
 * ascending entry order, padded with -1 when n_vis < k.
 * Arguments:
 *   qI e4m3 [Q, H_I, d_I]; qI_scale, w fp32 [Q, H_I]; kI e4m3 [ent_rows, d_I];
 *   kI_scale fp32 [ent_rows] (ent_rows: rows in kI / kI_scale; every visible entry's row
 *   ent_off[b] + i must be < ent_rows, else CSA_DEV_OOB and the rest are skipped); seq_len, ent_off int64 [B]; q_seq, q_pos int32 [Q]
 *   H_I in 1..64, d_I in {64, 128}, m >= 1 (4 for CSA), 1 <= k <= 2048
 *   max_n: upper bound of n_vis over the batch (sizes the workspace)
 *   idx_out int32 [Q, k]
 *   scores_out: nullable fp32 [Q, ld_scores] receiving s_i for i < n_vis (ld_scores >= max_n)
 *   workspace: device buffer of at least csa_indexer_workspace_size(Q, max_n, k) bytes,
 *   256-byte aligned; contents on entry are ignored.  It holds the largest score of every
 *   32 consecutive entries of every query (which the selection starts from), then the score
 *   rows.  With scores_out given the score rows go there: the workspace may then be just
 *   large enough for the first part (ceil(Q * ceil(max_n / 32) * 4 / 256) * 256 bytes), or
 *   NULL (with workspace_bytes 0), in which case the selection reads the full score rows.
 *   layout: nullable cache layout; with a block table the key rows (and kI_scale) follow
 *   it, block by block.
 * kI and qI must be 16-byte aligned.  Errors as above; CSA_DEV_NAN, CSA_DEV_CAPACITY.
 */
size_t csa_indexer_workspace_size(int32_t Q, int32_t max_n, int32_t k);
csa_status_t lightning_indexer_topk(const uint8_t* qI, const float* qI_scale, const float* w,
                                    const uint8_t* kI, const float* kI_scale, int64_t ent_rows,
                                    const int64_t* seq_len, const int64_t* ent_off,
                                    const int32_t* q_seq,
                                    const int32_t* q_pos, int32_t Q, int32_t B, int32_t H_I,
                                    int32_t d_I, int32_t m, int32_t k, int32_t max_n,
                                    int32_t* idx_out, float* scores_out, int64_t ld_scores,
                                    void* workspace, size_t workspace_bytes,
                                    const csa_cache_layout_t* layout, int32_t* dev_status,
                                    void* stream);

/*
 * lightning_indexer_topk_mxfp4 -- steps a3 + a4 with MXFP4 query heads and keys and,
 * optionally, BF16-rounded selector scores ("DeepSeek-V4 深度分析报告" Figure 2, "Lightning
 * Indexer FP4 Precision"; "其他注意力技术细节": the indexer computes in FP4; section 3.4:
 * MXFP4 quantisation on the QK path of CSA, the indexer scores quantised from FP32 to BF16
 * for the top-k selector).
 *   MXFP4 is the OCP microscaling format: e2m1 elements (+-{0, 0.5, 1, 1.5, 2, 3, 4, 6}),
 *   two per byte with element 2j in the low nibble, and one UE8M0 scale byte (2^(e-127),
 *   0xFF = NaN) per 32 consecutive elements.
 *   s_i = sum_h w_h * ReLU(q_h . k_i) over h ascending by fmaf in fp32, q_h . k_i the
 *   block-scaled dot product accumulated in fp32 by the tensor cores (exact when the
 *   blocks' partial sums are: the integer-valued inputs of the tests).  No per-head or
 *   per-entry factor besides w: the block scales carry the magnitudes.
 *   select_bf16 = 1: every score is rounded to BF16 (nearest, ties to even) and the top-k
 *   is taken on the rounded values with the same order (larger first, lower index first
 *   among equal values); the score rows then hold the rounded values (as fp32).  The
 *   section 3.4 reading: this variant trades the FP32 selection's bit-exact index set for a
 *   recall figure (the pages quote 99.7 % of the entries kept).  select_bf16 = 0 selects on
 *   the FP32 scores exactly as lightning_indexer_topk does.
 * Arguments: as lightning_indexer_topk, with
 *   qI uint8 [Q, H_I, d_I / 2] packed e2m1; qI_sf uint8 [Q, H_I, d_I / 32] UE8M0;
 *   w fp32 [Q, H_I]; kI uint8 [ent_rows, d_I / 2]; kI_sf uint8 [ent_rows, d_I / 32];
 *   H_I in {16, 32, 64}, d_I = 128.  qI, kI 16-byte aligned; qI_sf, kI_sf 4-byte aligned.
 *   The workspace is csa_indexer_workspace_size(Q, max_n, k) bytes, used as by
 *   lightning_indexer_topk.
 * Errors as lightning_indexer_topk.
 */
csa_status_t lightning_indexer_topk_mxfp4(const uint8_t* qI, const uint8_t* qI_sf,
                                          const float* w, const uint8_t* kI,
                                          const uint8_t* kI_sf, int64_t ent_rows,
                                          const int64_t* seq_len, const int64_t* ent_off,
                                          const int32_t* q_seq, const int32_t* q_pos, int32_t Q,
                                          int32_t B, int32_t H_I, int32_t d_I, int32_t m,
                                          int32_t k, int32_t max_n, int32_t select_bf16,
                                          int32_t* idx_out, float* scores_out,
                                          int64_t ld_scores, void* workspace,
                                          size_t workspace_bytes,
                                          const csa_cache_layout_t* layout,
                                          int32_t* dev_status, void* stream);

/*
 * csa_cache_append -- one decode token per sequence into the hybrid cache
 * ("DeepSeek-V4 深度分析报告" 3.5: the state cache holds the window's KV and the tokens not
 * yet compressed; the classical cache holds the entries in blocks of 128 tokens).
 *   For every sequence b, with p = seq_len[b] on entry: the token's raw KV and gate rows
 *   (kv_new, gate_new bf16 [B, D]) are written to its state-cache row (kv_off[b] + p mod
 *   kv_ring with a ring in the layout, else kv_off[b] + p - kv_pos0[b]; the row must be
 *   < kv_rows); if p + 1 is a multiple of m, the entry (p + 1) / m - 1 it completes gets its
 *   indexer key row kI_new[b] (e4m3 [B, d_I]) and scale kI_scale_new[b] written to the key
 *   store (kI [ent_rows, d_I], kI_scale [ent_rows]) at the entry's row (block table or
 *   ent_off; kI_new may be NULL to skip); then seq_len[b] = p + 1.  The entry itself is
 *   then compressed by csa_compress (with the same layout), after this call.
 *   A row outside kv_rows / ent_rows sets CSA_DEV_OOB and leaves seq_len[b] unchanged.
 *   The kernels after this call on the stream start only when it has completed.
 * Errors: CSA_ERR_INVALID_ARG, CSA_ERR_UNSUPPORTED (D), CSA_ERR_CUDA.
 */
csa_status_t csa_cache_append(const void* kv_new, const void* gate_new, const uint8_t* kI_new,
                              const float* kI_scale_new, int32_t d_I, int64_t* seq_len,
                              const int64_t* kv_off, const int64_t* kv_pos0, int64_t kv_rows,
                              const int64_t* ent_off, int64_t ent_rows, int32_t B, int32_t D,
                              int32_t m, void* kv, void* gate, uint8_t* kI, float* kI_scale,
                              const csa_cache_layout_t* layout, int32_t* dev_status,
                              void* stream);

/*
 * Context-parallel decode (the stuffyNLP post's context parallelism applied to the
 * selection and attention of "DeepSeek-V4 深度分析报告" 2.1 CSA).  A sequence's entries
 * are split into W contiguous slices (say one per GPU, slice r on rank r, slices in
 * ascending entry order), and a rank holds the key and entry rows of its slice only.  One
 * decode step: each rank selects its slice's top-k with lightning_indexer_topk (with
 * scores_out), csa_cp_candidates turns that into candidates, the ranks' candidates are
 * gathered (slice-major), csa_topk_merge selects the sequence's top-k from them,
 * csa_cp_pack_rows writes the selected rows this rank holds, an integer sum over the
 * ranks' packed buffers gathers every selected row, and sparse_mqa_attn runs over them.
 * Since the order within a slice is the order of the whole sequence, every entry of the
 * sequence's top-k is in its slice's top-k; the merge uses the order of the selection
 * (larger score first, lower entry index first among equal scores, -0 = +0) and writes the
 * same output (ascending entry order, -1 padded), so the index set is bit for bit the one
 * lightning_indexer_topk selects over the whole sequence.
 *
 * csa_cp_candidates -- a slice's selection as candidates of the whole sequence.
 *   idx int32 [Q, k]: lightning_indexer_topk's output over the slice (indices within the
 *   slice, -1 padded); scores fp32 [Q, ld_scores]: its scores_out rows; q_seq int32 [Q];
 *   slice_lo int64 [B]: the slice's first entry of each sequence.  Writes cand_idx int32
 *   [Q, k] = idx + slice_lo[q_seq] (-1 kept) and cand_scores fp32 [Q, k] = the entry's
 *   score (0 for -1).  An index >= ld_scores, a sum above INT32_MAX or a q_seq outside
 *   0..B-1 sets CSA_DEV_OOB and gives -1.
 *
 * csa_topk_merge -- the sequence's top-k from the W slices' candidates.
 *   cand_scores fp32, cand_idx int32: candidate j of slice r for query q at element
 *     r * slice_stride + q * k_in + j (so [W, Q, k_in] with slice_stride = Q * k_in, the
 *     layout a gather of every rank's [Q, k_in] gives), slices in ascending entry order,
 *     each slice's set ascending (as csa_cp_candidates writes them) -- so the candidates
 *     are in ascending entry order.  -1 = no candidate.  1 <= W * k_in <= 16384.
 *   k in 1..2048; idx_out int32 [Q, k].
 *   A NaN score sets CSA_DEV_NAN.
 *
 * csa_cp_pack_rows -- the selected rows this rank holds, at their output positions.
 *   idx int32 [Q, k]: the merged selection (entry indices of the whole sequence); q_seq
 *   int32 [Q]; slice_lo, slice_n int64 [B]: this rank's slice of each sequence (entries
 *   slice_lo .. slice_lo + slice_n - 1); ent_off int64 [B]: where each sequence's slice
 *   starts in `entries` (this rank's store, ent_rows rows of row_bytes bytes, as
 *   csa_entry_row_bytes gives; row_bytes a multiple of 16).  Writes out uint8 [Q, k,
 *   row_bytes]: row (q, j) is the entry row of idx[q, j] if this rank's slice holds it, else
 *   zeros.  Every position has exactly one rank with its row, so the element-wise integer
 *   sum of the W ranks' buffers (say NCCL all_reduce on an int32 view) is the gathered
 *   [Q * k, row_bytes] store that sparse_mqa_attn reads with entry indices 0..k-1 of query
 *   q at rows q * k ... (ent_off = q * k for one query per sequence).  local_idx
 *   (nullable) int32 [Q, k] receives those indices: j where idx[q, j] >= 0, else -1.  A
 *   row outside 0..ent_rows-1 sets CSA_DEV_OOB and is written as zeros.  entries and out
 *   16-byte aligned.
 * Errors (all three): CSA_ERR_INVALID_ARG, CSA_ERR_UNSUPPORTED, CSA_ERR_CUDA.
 */
csa_status_t csa_cp_candidates(const int32_t* idx, const float* scores, int64_t ld_scores,
                               const int32_t* q_seq, const int64_t* slice_lo, int32_t Q,
                               int32_t B, int32_t k, int32_t* cand_idx, float* cand_scores,
                               int32_t* dev_status, void* stream);
csa_status_t csa_topk_merge(const float* cand_scores, const int32_t* cand_idx,
                            int64_t slice_stride, int32_t W, int32_t Q, int32_t k_in, int32_t k,
                            int32_t* idx_out, int32_t* dev_status, void* stream);
csa_status_t csa_cp_pack_rows(const int32_t* idx, const int32_t* q_seq, const int64_t* slice_lo,
                              const int64_t* slice_n, const int64_t* ent_off,
                              const uint8_t* entries, int64_t ent_rows, int32_t row_bytes,
                              int32_t Q, int32_t B, int32_t k, uint8_t* out,
                              int32_t* local_idx, int32_t* dev_status, void* stream);

/*
 * sparse_mqa_attn -- CSA shared-KV MQA over the selected entries and the window (a5).
 *   "DeepSeek-V4 深度分析报告" 2.1 CSA (top-k entries plus a 128-token sliding window);
 *   "其他注意力技术细节": Shared Key-Value MQA (an entry is both key and value, all heads
 *   share it), Partial RoPE with inverse RoPE on the output, Attention Sink (learnable
 *   per-head logit, weights may sum to less than 1).
 * For query q (sequence b, position t) and head h:
 *   keys K = { entry idx[q,j] : idx >= 0 }  U  { window rows p = max(0,t-W+1) .. t },
 *   window row p = RoPE_p(RMSNorm(kv[p])) computed on the fly in fp32 (never stored);
 *   l_j = softmax_scale * < RoPE_t(q[q,h]), k_j >,  M = max(sink[h], max_j l_j),
 *   o = sum_j e^(l_j-M) k_j / (e^(sink[h]-M) + sum_j e^(l_j-M)),  out = RoPE_{-t}(o) (bf16).
 * Arguments:
 *   q bf16 [Q, H, D]; entries in format fmt, ent_rows rows (an entry row ent_off[b] + i at or
 *   past ent_rows sets CSA_DEV_OOB and is skipped); kv bf16 raw rows for the window;
 *   idx int32 [Q, k] (entries < n_vis(t) for ratio m, or -1 = skip); sink fp32 [H]
 *   H in {16, 64, 128}; D 128 (bf16) or 576 (either format); 0 <= W <= 128
 *   out bf16 [Q, H, D]
 *   layout: nullable cache layout (the selected entries' rows through a block table; the
 *   window's raw rows through a state-cache ring)
 * Pointers q/kv/entries/out must be 16-byte aligned.  Out-of-range indices set CSA_DEV_OOB
 * and are skipped.
 */
csa_status_t sparse_mqa_attn(const void* q, const void* entries, int32_t fmt, int64_t ent_rows,
                             const int64_t* seq_len, const int64_t* ent_off, const void* kv,
                             const int64_t* kv_off,
                             const int64_t* kv_pos0, const int32_t* q_seq,
                             const int32_t* q_pos, const int32_t* idx, int32_t k, int32_t m,
                             const float* sink, int32_t Q, int32_t B, int32_t H, int32_t D,
                             int32_t W, float softmax_scale, float rope_theta, float eps,
                             void* out, const csa_cache_layout_t* layout, int32_t* dev_status,
                             void* stream);

/*
 * dense_hca_attn -- HCA dense MQA over every visible entry plus the window (a6).
 *   "DeepSeek-V4 深度分析报告" 2.1 HCA: dense attention over all compressed entries, with
 *   the same sliding-window branch; Figure 2 "Dense Attention on All Compressed KV
 *   Entries".  As sparse_mqa_attn with K = { entries 0 .. n_vis(t)-1 } U window, where
 *   n_vis(t) = floor((t+1)/m) (m = 128 for HCA).
 *   max_n: upper bound of n_vis over the batch; workspace: at least
 *   dense_hca_workspace_size(Q, H, D, max_n) bytes, 256-byte aligned (partial softmax
 *   states of the fixed entry chunks one query is split into; the chunking depends only
 *   on the query's own n_vis and the shape, so results do not depend on the batch).
 */
size_t dense_hca_workspace_size(int32_t Q, int32_t H, int32_t D, int32_t max_n);
/* layout: nullable; its kv_ring applies to the window, a block table is refused (the dense
 * pass reads each sequence's entries as one contiguous array). */
csa_status_t dense_hca_attn(const void* q, const void* entries, int32_t fmt, int64_t ent_rows,
                            const int64_t* seq_len, const int64_t* ent_off, const void* kv,
                            const int64_t* kv_off,
                            const int64_t* kv_pos0, const int32_t* q_seq, const int32_t* q_pos,
                            int32_t m, const float* sink, int32_t Q, int32_t B, int32_t H,
                            int32_t D, int32_t W, float softmax_scale, float rope_theta,
                            float eps, int32_t max_n, void* out, void* workspace,
                            size_t workspace_bytes, const csa_cache_layout_t* layout,
                            int32_t* dev_status, void* stream);

/*
 * lightning_indexer_topk_noalloc -- the same scores and selection as
 * lightning_indexer_topk, for callers that cannot allocate device memory (no counterpart
 * on the pages: it is a deployment variant of this library).
 *   Some callers cannot call cudaMalloc or provide a workspace: a plugin inside a host
 *   framework that owns the whole device-memory pool and gives plugins no scratch, or a
 *   latency-critical loop where a cudaMalloc (which may synchronise the device) is not
 *   allowed.  This call takes the same inputs and outputs minus the workspace and keeps
 *   its scratch (the per-query score rows) in a device array inside the library of
 *   CSA_NOALLOC_SCRATCH_BYTES bytes; it allocates nothing.
 *   - A call needing more than that (csa_indexer_workspace_size(Q, max_n, k) > the size)
 *     returns CSA_ERR_WORKSPACE with a message and launches nothing.  16 MiB covers, e.g.,
 *     32 queries of up to 127072 visible entries.  With scores_out given, the scores are
 *     written there, the array is not used and there is no such limit.
 *   - Every GPU that loads the library holds the array until the process exits.
 *   - All calls on a device share the array, which keeps the last call's contents;
 *     nothing in it has to start at zero.  Calls whose kernels overlap on the GPU (e.g.
 *     on two unordered streams) race on it: order them on one stream.
 *   - Each call made outside stream capture resolves the array's device address on the
 *     current device (cudaGetSymbolAddress) and caches it; a call made while `stream` is
 *     being captured uses the cached address.  So make one call on each device before any
 *     stream capture, and again after a cudaDeviceReset (which invalidates the address).
 */
#define CSA_NOALLOC_SCRATCH_BYTES (16u << 20)
csa_status_t lightning_indexer_topk_noalloc(const uint8_t* qI, const float* qI_scale,
                                            const float* w, const uint8_t* kI,
                                            const float* kI_scale, int64_t ent_rows,
                                            const int64_t* seq_len,
                                            const int64_t* ent_off, const int32_t* q_seq,
                                            const int32_t* q_pos, int32_t Q, int32_t B,
                                            int32_t H_I, int32_t d_I, int32_t m, int32_t k,
                                            int32_t max_n, int32_t* idx_out, float* scores_out,
                                            int64_t ld_scores, int32_t* dev_status, void* stream);

/*
 * Launch accounting and kernel timing (no counterpart on the pages; instrumentation).
 *   csa_launch_count: kernels this library has launched in the process so far.
 *   csa_profile_enable(1): from now on every launch is bracketed by a CUDA event pair
 *     recorded on its own stream (adds two event records per launch); 0 turns it off.
 *   csa_profile_collect: waits for the recorded events, writes one record per kernel
 *     kind timed since the last collect (launch count and total device milliseconds) to
 *     out[0 .. max_entries), returns how many it wrote, and resets the totals.  With
 *     keep_pending != 0 the event pairs stay registered: launches captured into a CUDA
 *     graph record the same events on every replay, so a collect after each replay reads
 *     that replay's kernel times.
 * Thread-safe.  Uses the CUDA device that was current at each launch.
 */
typedef struct {
    char name[40];
    long long launches;
    double total_ms;
} csa_kernel_time_t;
long long csa_launch_count(void);
void csa_profile_enable(int on);
int csa_profile_collect(csa_kernel_time_t* out, int max_entries, int keep_pending);

/*
 * csa_debug_set_wait_limit -- test hook for the device-side failure path (no counterpart
 * on the pages).
 *   Every wait of the tensor-core kernels on an mbarrier is bounded: past the limit it
 *   flags CSA_DEV_TIMEOUT in dev_status and the CTA winds down (it waits for its own
 *   copies and MMAs in flight, frees its tensor memory and returns).  This call sets that
 *   limit, in SM clock cycles, for every kernel of the library; cycles <= 0 restores the
 *   default of 4e9 cycles (about 2 s).  The drains of a CTA's own copies and MMAs always
 *   keep the default.  A limit of a few hundred cycles makes waits give up at once, so a
 *   test can check that the timeout path reports CSA_DEV_TIMEOUT and that later calls are
 *   exact again.  Lower it only around kernels launched without thread-block clusters.
 *   Unlike the other calls, this one copies to device memory synchronously: call it with
 *   no libcsa kernel in flight and never during stream capture.
 * Errors: CSA_ERR_CUDA.
 */
csa_status_t csa_debug_set_wait_limit(long long cycles);

#ifdef __cplusplus
}
#endif
#endif /* CSA_H */
