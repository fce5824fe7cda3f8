// The C ABI of libcsa: host-side validation, workspace layout and kernel dispatch.
// Declarations and the contract of every call are in include/csa.h.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "launchers.cuh"



namespace {

thread_local char g_err[512] = "";

csa_status_t fail(csa_status_t s, const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
    return s;
}

csa_status_t ok() {
    g_err[0] = '\0';
    return CSA_OK;
}

csa_status_t cuda_status(cudaError_t e, const char* what) {
    if (e == cudaSuccess) return ok();
    return fail(CSA_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return ((uintptr_t)p % a) == 0; }

#define REQUIRE(cond, ...)                                      \
    do {                                                        \
        if (!(cond)) return fail(CSA_ERR_INVALID_ARG, __VA_ARGS__); \
    } while (0)
#define SUPPORT(cond, ...)                                      \
    do {                                                        \
        if (!(cond)) return fail(CSA_ERR_UNSUPPORTED, __VA_ARGS__); \
    } while (0)

size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Workspace of lightning_indexer_topk: first the group maxima (the largest score key of
// every 32 consecutive entries of every query, which the top-k selects from), then the
// score rows (round_up(max_n, 32) floats per query), which scores_out replaces.
struct IndexerWorkspace {
    int64_t ld, ld_g;
    size_t gmax_bytes, off_scores, total;
};
IndexerWorkspace indexer_workspace(int32_t Q, int32_t max_n) {
    IndexerWorkspace w;
    w.ld = (int64_t)round_up((size_t)max_n, 32);
    w.ld_g = w.ld / 32;
    w.gmax_bytes = round_up((size_t)Q * w.ld_g * 4, 256);
    w.off_scores = w.gmax_bytes;
    w.total = w.off_scores + round_up((size_t)Q * w.ld * sizeof(float), 256) + 256;
    return w;
}

// Entry and raw-row maps of a call.  A block table needs m = 4 (blocks of 128 tokens = 32
// CSA entries); without one, entries are contiguous from ent_off.  A ring makes kv_pos0
// unused.
csa_status_t make_rows(const csa_cache_layout_t* L, int m, const int64_t* ent_off,
                       const int64_t* kv_off, const int64_t* kv_pos0, bool need_raw,
                       csa::EntryRows* er, csa::RawRows* raw, bool need_ent = true) {
    const int32_t* bt = L ? L->block_table : nullptr;
    const int64_t ring = L ? L->kv_ring : 0;
    REQUIRE(!bt || (m == 4 && L->bt_stride >= 1),
            "a block table needs m = 4 (blocks of 32 entries) and bt_stride >= 1");
    REQUIRE(!need_ent || bt || ent_off, "ent_off must not be null without a block table");
    REQUIRE(ring >= 0, "kv_ring must be >= 0");
    if (need_raw) {
        REQUIRE(kv_off && (ring > 0 || kv_pos0), "kv_off (and kv_pos0 without a ring) must not be null");
    }
    er->ent_off = ent_off;
    er->bt = bt;
    er->bt_stride = bt ? L->bt_stride : 0;
    er->pe_shift = 5;
    raw->kv_off = kv_off;
    raw->kv_pos0 = kv_pos0;
    raw->ring = ring;
    return ok();
}

csa_status_t compress_common(int m, int span, const void* kv, const void* gate,
                             const float* bias, const int64_t* seq_len, const int64_t* kv_off, const int64_t* kv_pos0,
                             const int64_t* ent_off, const int32_t* item_seq,
                             const int32_t* item_ent, int64_t n_items, int32_t B, int32_t D,
                             int32_t fmt, float theta, float eps, void* entries,
                             const csa_cache_layout_t* layout, int32_t* dev_status,
                             void* stream) {
    REQUIRE(n_items >= 0 && n_items < (1ll << 31), "n_items out of range: %lld", (long long)n_items);
    if (n_items == 0) return ok();
    REQUIRE(kv && gate && bias && seq_len && item_seq && item_ent && entries,
            "null pointer argument");
    csa::EntryRows er;
    csa::RawRows raw;
    csa_status_t lv = make_rows(layout, m, ent_off, kv_off, kv_pos0, true, &er, &raw);
    if (lv != CSA_OK) return lv;
    REQUIRE(aligned(kv, 16) && aligned(gate, 16) && aligned(entries, 16) && aligned(bias, 16),
            "kv, gate, pos_bias and entries must be 16-byte aligned");
    REQUIRE(B >= 1, "B must be >= 1");
    REQUIRE(fmt == CSA_KV_BF16 || fmt == CSA_KV_FP8_576, "unknown entry format %d", fmt);
    SUPPORT(D == 128 || D == 576, "head dim %d not supported (128 or 576)", D);
    SUPPORT(fmt == CSA_KV_BF16 || D == 576, "fp8 entry format needs D = 576");
    REQUIRE(theta > 1.f && eps >= 0.f, "rope_theta must be > 1 and eps >= 0");
    cudaError_t e = csa::launch_compress(span, kv, gate, bias, seq_len, raw, er, item_seq,
                                         item_ent, n_items, B, m, D, fmt, theta, eps, entries,
                                         dev_status, (cudaStream_t)stream);
    return cuda_status(e, "compress launch");
}

}  // namespace

namespace csa {
void set_error_message(const char* fmt, ...) {
    va_list ap;
    va_start(ap, fmt);
    vsnprintf(g_err, sizeof(g_err), fmt, ap);
    va_end(ap);
}

namespace {
// Setters of the per-file wait limits, filled while the library loads (static
// initialisation of the kernel files), read by csa_debug_set_wait_limit.
constexpr int kMaxWaitLimitSetters = 16;
struct WaitLimitSetters {
    cudaError_t (*fn[kMaxWaitLimitSetters])(long long);
    int n;
};
WaitLimitSetters& wait_limit_setters() {
    static WaitLimitSetters s = {};
    return s;
}
}  // namespace

void register_wait_limit_setter(cudaError_t (*set)(long long cycles)) {
    WaitLimitSetters& s = wait_limit_setters();
    if (s.n < kMaxWaitLimitSetters) s.fn[s.n++] = set;
}
}  // namespace csa

extern "C" {

int csa_version(void) { return 100; }

csa_status_t csa_debug_set_wait_limit(long long cycles) {
    const long long c = cycles > 0 ? cycles : 4000000000LL;
    csa::WaitLimitSetters& s = csa::wait_limit_setters();
    if (s.n == 0) return fail(CSA_ERR_CUDA, "csa_debug_set_wait_limit: no kernel file registered");
    for (int i = 0; i < s.n; i++) {
        const cudaError_t e = s.fn[i](c);
        if (e != cudaSuccess) return cuda_status(e, "csa_debug_set_wait_limit");
    }
    return ok();
}

const char* csa_last_error(void) { return g_err; }

int32_t csa_entry_row_bytes(int32_t fmt, int32_t D) {
    if (fmt == CSA_KV_BF16 && (D == 128 || D == 576)) return 2 * D;
    if (fmt == CSA_KV_FP8_576 && D == 576) return 656;
    return -1;
}

csa_status_t csa_compress(const void* kv, const void* gate, const float* pos_bias,
                          const int64_t* seq_len, const int64_t* kv_off, const int64_t* kv_pos0,
                          const int64_t* ent_off,
                          const int32_t* item_seq, const int32_t* item_ent, int64_t n_items,
                          int32_t B, int32_t D, int32_t fmt, float rope_theta, float eps,
                          void* entries, const csa_cache_layout_t* layout, int32_t* dev_status,
                          void* stream) {
    return compress_common(4, 8, kv, gate, pos_bias, seq_len, kv_off, kv_pos0, ent_off, item_seq, item_ent,
                           n_items, B, D, fmt, rope_theta, eps, entries, layout, dev_status, stream);
}

csa_status_t hca_compress(const void* kv, const void* gate, const float* pos_bias,
                          const int64_t* seq_len, const int64_t* kv_off, const int64_t* kv_pos0,
                          const int64_t* ent_off,
                          const int32_t* item_seq, const int32_t* item_ent, int64_t n_items,
                          int32_t B, int32_t D, int32_t fmt, float rope_theta, float eps,
                          void* entries, const csa_cache_layout_t* layout, int32_t* dev_status,
                          void* stream) {
    return compress_common(128, 128, kv, gate, pos_bias, seq_len, kv_off, kv_pos0, ent_off, item_seq,
                           item_ent, n_items, B, D, fmt, rope_theta, eps, entries, layout,
                           dev_status, stream);
}

size_t csa_indexer_workspace_size(int32_t Q, int32_t max_n, int32_t k) {
    if (Q <= 0 || max_n < 0 || k <= 0) return 0;
    return indexer_workspace(Q, max_n).total;
}

csa_status_t lightning_indexer_topk(const uint8_t* qI, const float* qI_scale, const float* w,
                                    const uint8_t* kI, const float* kI_scale, int64_t ent_rows,
                                    const int64_t* seq_len, const int64_t* ent_off,
                                    const int32_t* q_seq,
                                    const int32_t* q_pos, int32_t Q, int32_t B, int32_t H_I,
                                    int32_t d_I, int32_t m, int32_t k, int32_t max_n,
                                    int32_t* idx_out, float* scores_out, int64_t ld_scores,
                                    void* workspace, size_t workspace_bytes,
                                    const csa_cache_layout_t* layout, int32_t* dev_status,
                                    void* stream) {
    REQUIRE(Q >= 0, "Q must be >= 0");
    if (Q == 0) return ok();
    REQUIRE(qI && qI_scale && w && seq_len && q_seq && q_pos && idx_out,
            "null pointer argument");
    csa::EntryRows er;
    csa::RawRows raw;
    csa_status_t lv = make_rows(layout, m, ent_off, nullptr, nullptr, false, &er, &raw);
    if (lv != CSA_OK) return lv;
    REQUIRE(max_n >= 0, "max_n must be >= 0");
    REQUIRE(ent_rows >= 0 && ent_rows < (1ll << 31), "ent_rows out of range");
    REQUIRE(max_n == 0 || ent_rows == 0 || (kI && kI_scale), "null key pointer");
    REQUIRE(aligned(qI, 16) && (kI == nullptr || aligned(kI, 16)), "qI and kI must be 16-byte aligned");
    REQUIRE(B >= 1 && m >= 1, "B and m must be >= 1");
    SUPPORT(H_I >= 1 && H_I <= 64, "indexer heads %d not supported (1..64)", H_I);
    SUPPORT(d_I == 64 || d_I == 128, "indexer dim %d not supported (64 or 128)", d_I);
    SUPPORT(k >= 1 && k <= 2048, "k = %d not supported (1..2048)", k);
    REQUIRE(scores_out == nullptr || ld_scores >= max_n, "ld_scores must be >= max_n");
    // With scores_out the score rows go there and the workspace needs only its group-maxima
    // region (a smaller or missing workspace then leaves the top-k to the full rows).
    const IndexerWorkspace L = indexer_workspace(Q, max_n);
    if (!scores_out && (!workspace || workspace_bytes < L.total || !aligned(workspace, 256)))
        return fail(CSA_ERR_WORKSPACE, "workspace must be >= %zu bytes, 256-byte aligned", L.total);
    float* scores = scores_out ? scores_out : (float*)((uint8_t*)workspace + L.off_scores);
    const int64_t ld = scores_out ? ld_scores : L.ld;
    cudaStream_t s = (cudaStream_t)stream;
    cudaError_t e;
    uint32_t* gmax = nullptr;
    // every supported shape runs on the tensor cores (head counts padded to 16, 32 or 64)
    if (workspace && workspace_bytes >= L.gmax_bytes && aligned(workspace, 256))
        gmax = (uint32_t*)workspace;
    e = csa::launch_indexer_tc(qI, qI_scale, w, kI, kI_scale, ent_rows, seq_len, er, q_seq, q_pos,
                               Q, B, H_I, d_I, m, max_n, scores, ld, dev_status, s, gmax, L.ld_g);
    if (e != cudaSuccess) return cuda_status(e, "indexer launch");
    e = csa::launch_topk(scores, ld, q_seq, q_pos, seq_len, Q, B, m, max_n, k, idx_out, dev_status,
                         s, gmax, L.ld_g);
    return cuda_status(e, "top-k launch");
}

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
                                          int32_t* dev_status, void* stream) {
    REQUIRE(Q >= 0, "Q must be >= 0");
    if (Q == 0) return ok();
    REQUIRE(qI && qI_sf && w && seq_len && q_seq && q_pos && idx_out,
            "null pointer argument");
    csa::EntryRows er;
    csa::RawRows raw;
    csa_status_t lv = make_rows(layout, m, ent_off, nullptr, nullptr, false, &er, &raw);
    if (lv != CSA_OK) return lv;
    REQUIRE(max_n >= 0, "max_n must be >= 0");
    REQUIRE(ent_rows >= 0 && ent_rows < (1ll << 31), "ent_rows out of range");
    REQUIRE(max_n == 0 || ent_rows == 0 || (kI && kI_sf), "null key pointer");
    REQUIRE(aligned(qI, 16) && (kI == nullptr || aligned(kI, 16)), "qI and kI must be 16-byte aligned");
    REQUIRE(aligned(qI_sf, 4) && (kI_sf == nullptr || aligned(kI_sf, 4)),
            "qI_sf and kI_sf must be 4-byte aligned");
    REQUIRE(B >= 1 && m >= 1, "B and m must be >= 1");
    REQUIRE(select_bf16 == 0 || select_bf16 == 1, "select_bf16 must be 0 or 1");
    SUPPORT(csa::indexer_fp4_supported(H_I, d_I),
            "MXFP4 indexer shape H_I = %d, d_I = %d not supported (16, 32 or 64 heads; d_I = 128)",
            H_I, d_I);
    SUPPORT(k >= 1 && k <= 2048, "k = %d not supported (1..2048)", k);
    REQUIRE(scores_out == nullptr || ld_scores >= max_n, "ld_scores must be >= max_n");
    const IndexerWorkspace L = indexer_workspace(Q, max_n);
    if (!scores_out && (!workspace || workspace_bytes < L.total || !aligned(workspace, 256)))
        return fail(CSA_ERR_WORKSPACE, "workspace must be >= %zu bytes, 256-byte aligned", L.total);
    float* scores = scores_out ? scores_out : (float*)((uint8_t*)workspace + L.off_scores);
    const int64_t ld = scores_out ? ld_scores : L.ld;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t* gmax = nullptr;
    if (workspace && workspace_bytes >= L.gmax_bytes && aligned(workspace, 256))
        gmax = (uint32_t*)workspace;
    cudaError_t e = csa::launch_indexer_fp4(qI, qI_sf, w, kI, kI_sf, ent_rows, seq_len, er,
                                            q_seq, q_pos, Q, B, H_I, m, max_n, select_bf16,
                                            scores, ld, dev_status, s, gmax, L.ld_g);
    if (e != cudaSuccess) return cuda_status(e, "MXFP4 indexer launch");
    e = csa::launch_topk(scores, ld, q_seq, q_pos, seq_len, Q, B, m, max_n, k, idx_out, dev_status,
                         s, gmax, L.ld_g);
    return cuda_status(e, "top-k launch");
}

csa_status_t csa_cache_append(const void* kv_new, const void* gate_new, const uint8_t* kI_new,
                              const float* kI_scale_new, int32_t d_I, int64_t* seq_len,
                              const int64_t* kv_off, const int64_t* kv_pos0, int64_t kv_rows,
                              const int64_t* ent_off, int64_t ent_rows, int32_t B, int32_t D,
                              int32_t m, void* kv, void* gate, uint8_t* kI, float* kI_scale,
                              const csa_cache_layout_t* layout, int32_t* dev_status,
                              void* stream) {
    REQUIRE(B >= 0, "B must be >= 0");
    if (B == 0) return ok();
    REQUIRE(kv_new && gate_new && seq_len && kv && gate, "null pointer argument");
    REQUIRE(aligned(kv_new, 16) && aligned(gate_new, 16) && aligned(kv, 16) && aligned(gate, 16),
            "kv_new, gate_new, kv and gate must be 16-byte aligned");
    SUPPORT(D == 128 || D == 576, "head dim %d not supported (128 or 576)", D);
    REQUIRE(m >= 1 && kv_rows >= 0 && ent_rows >= 0, "bad m / kv_rows / ent_rows");
    if (kI_new) {
        REQUIRE(kI_scale_new && kI && kI_scale, "null indexer-key pointer");
        REQUIRE(d_I == 64 || d_I == 128, "d_I must be 64 or 128");
        REQUIRE(aligned(kI_new, 16) && aligned(kI, 16), "kI_new and kI must be 16-byte aligned");
    }
    csa::EntryRows er;
    csa::RawRows raw;
    csa_status_t v = make_rows(layout, m, ent_off, kv_off, kv_pos0, true, &er, &raw,
                               kI_new != nullptr);
    if (v != CSA_OK) return v;
    return cuda_status(csa::launch_cache_append((const uint16_t*)kv_new, (const uint16_t*)gate_new,
                                                kI_new, kI_scale_new, seq_len, raw, er, B, D, d_I,
                                                m, kv_rows, ent_rows, (uint16_t*)kv,
                                                (uint16_t*)gate, kI, kI_scale, dev_status,
                                                (cudaStream_t)stream),
                       "cache append launch");
}

csa_status_t csa_topk_merge(const float* cand_scores, const int32_t* cand_idx,
                            int64_t slice_stride, int32_t W, int32_t Q, int32_t k_in, int32_t k,
                            int32_t* idx_out, int32_t* dev_status, void* stream) {
    REQUIRE(Q >= 0, "Q must be >= 0");
    if (Q == 0) return ok();
    REQUIRE(cand_scores && cand_idx && idx_out, "null pointer argument");
    REQUIRE(W >= 1 && k_in >= 1, "W and k_in must be >= 1");
    REQUIRE(W == 1 || slice_stride >= (int64_t)Q * k_in,
            "slice_stride %lld < Q * k_in", (long long)slice_stride);
    SUPPORT(k >= 1 && k <= 2048, "k = %d not supported (1..2048)", k);
    SUPPORT((int64_t)W * k_in <= (1 << 30) && csa::topk_merge_supported(W * k_in, k),
            "W * k_in = %lld not supported (1..16384 candidates per query)",
            (long long)W * k_in);
    return cuda_status(csa::launch_topk_merge(cand_scores, cand_idx, slice_stride, W, Q, k_in,
                                              k, idx_out, dev_status, (cudaStream_t)stream),
                       "top-k merge launch");
}

csa_status_t csa_cp_candidates(const int32_t* idx, const float* scores, int64_t ld_scores,
                               const int32_t* q_seq, const int64_t* slice_lo, int32_t Q,
                               int32_t B, int32_t k, int32_t* cand_idx, float* cand_scores,
                               int32_t* dev_status, void* stream) {
    REQUIRE(Q >= 0 && k >= 1 && B >= 1, "need Q >= 0, k >= 1, B >= 1");
    if (Q == 0) return ok();
    REQUIRE(idx && scores && q_seq && slice_lo && cand_idx && cand_scores,
            "null pointer argument");
    REQUIRE(ld_scores >= 1, "ld_scores must be >= 1");
    return cuda_status(csa::launch_cp_candidates(idx, scores, ld_scores, q_seq, slice_lo, Q, B,
                                                 k, cand_idx, cand_scores, dev_status,
                                                 (cudaStream_t)stream),
                       "candidate launch");
}

csa_status_t csa_cp_pack_rows(const int32_t* idx, const int32_t* q_seq, const int64_t* slice_lo,
                              const int64_t* slice_n, const int64_t* ent_off,
                              const uint8_t* entries, int64_t ent_rows, int32_t row_bytes,
                              int32_t Q, int32_t B, int32_t k, uint8_t* out,
                              int32_t* local_idx, int32_t* dev_status, void* stream) {
    REQUIRE(Q >= 0 && k >= 1 && B >= 1, "need Q >= 0, k >= 1, B >= 1");
    if (Q == 0) return ok();
    REQUIRE(idx && q_seq && slice_lo && slice_n && ent_off && entries && out,
            "null pointer argument");
    REQUIRE(row_bytes >= 16 && row_bytes % 16 == 0, "row_bytes must be a positive multiple of 16");
    REQUIRE(aligned(entries, 16) && aligned(out, 16), "entries and out must be 16-byte aligned");
    REQUIRE(ent_rows >= 0, "ent_rows must be >= 0");
    return cuda_status(csa::launch_cp_pack_rows(idx, q_seq, slice_lo, slice_n, ent_off, entries,
                                                ent_rows, row_bytes, Q, B, k, out, local_idx,
                                                dev_status, (cudaStream_t)stream),
                       "row pack launch");
}

static csa_status_t attn_validate(const void* q, const void* entries, int32_t fmt, int64_t ent_rows,
                                  const int64_t* seq_len, const int64_t* ent_off, const void* kv, const int64_t* kv_off,
                                  const int64_t* kv_pos0, const int32_t* q_seq,
                                  const int32_t* q_pos, const float* sink, int32_t B,
                                  int32_t H, int32_t D, int32_t W, int32_t m, float scale,
                                  float theta, float eps, void* out) {
    REQUIRE(q && entries && seq_len && kv && q_seq && q_pos && sink && out,
            "null pointer argument");
    REQUIRE(aligned(q, 16) && aligned(entries, 16) && aligned(kv, 16) && aligned(out, 16),
            "q, entries, kv and out must be 16-byte aligned");
    REQUIRE(fmt == CSA_KV_BF16 || fmt == CSA_KV_FP8_576, "unknown entry format %d", fmt);
    SUPPORT(D == 128 || D == 576, "head dim %d not supported (128 or 576)", D);
    SUPPORT(fmt == CSA_KV_BF16 || D == 576, "fp8 entry format needs D = 576");
    SUPPORT(H == 16 || H == 64 || H == 128, "query heads %d not supported (16, 64, 128)", H);
    REQUIRE(W >= 0 && W <= 128, "window %d outside 0..128", W);
    REQUIRE(ent_rows >= 0 && ent_rows < (1ll << 31), "ent_rows out of range");
    REQUIRE(B >= 1 && m >= 1, "B and m must be >= 1");
    REQUIRE(scale > 0.f && theta > 1.f && eps >= 0.f, "bad softmax_scale / rope_theta / eps");
    return ok();
}

csa_status_t sparse_mqa_attn(const void* q, const void* entries, int32_t fmt, int64_t ent_rows,
                             const int64_t* seq_len, const int64_t* ent_off, const void* kv, const int64_t* kv_off,
                             const int64_t* kv_pos0, const int32_t* q_seq,
                             const int32_t* q_pos, const int32_t* idx, int32_t k, int32_t m,
                             const float* sink, int32_t Q, int32_t B, int32_t H, int32_t D,
                             int32_t W, float softmax_scale, float rope_theta, float eps,
                             void* out, const csa_cache_layout_t* layout, int32_t* dev_status,
                             void* stream) {
    REQUIRE(Q >= 0, "Q must be >= 0");
    if (Q == 0) return ok();
    csa_status_t v = attn_validate(q, entries, fmt, ent_rows, seq_len, ent_off, kv, kv_off, kv_pos0, q_seq, q_pos,
                                   sink, B, H, D, W, m, softmax_scale, rope_theta, eps, out);
    if (v != CSA_OK) return v;
    REQUIRE(idx != nullptr, "idx must not be null");
    SUPPORT(k >= 1 && k <= 2048, "k = %d not supported (1..2048)", k);
    csa::EntryRows er;
    csa::RawRows raw;
    v = make_rows(layout, m, ent_off, kv_off, kv_pos0, true, &er, &raw);
    if (v != CSA_OK) return v;
    csa::AttnArgs a{(const uint16_t*)q, (const uint8_t*)entries, er, (const uint16_t*)kv,
                    raw, q_seq, q_pos, seq_len, idx, ent_rows, sink, (uint16_t*)out, dev_status,
                    k, m, B, H, W, fmt, softmax_scale, eps, log2((double)rope_theta)};
    if (csa::attn_tc_supported(H, D, fmt))
        return cuda_status(csa::launch_attn_tc(a, Q, 0, nullptr, (cudaStream_t)stream),
                           "attention launch");
    if (csa::attn576_tc_supported(H, D, fmt))
        return cuda_status(csa::launch_attn576_tc(a, Q, (cudaStream_t)stream), "attention launch");
    return cuda_status(csa::launch_attn_simt(a, Q, D, (cudaStream_t)stream), "attention launch");
}

size_t dense_hca_workspace_size(int32_t Q, int32_t H, int32_t D, int32_t max_n) {
    if (Q <= 0 || max_n < 0) return 256;
    size_t need = 0;
    if (csa::attn_tc_supported(H, D, CSA_KV_BF16)) need = csa::attn_tc_workspace_bytes(Q, max_n);
    return round_up(need, 256) + 256;
}

csa_status_t dense_hca_attn(const void* q, const void* entries, int32_t fmt, int64_t ent_rows,
                            const int64_t* seq_len, const int64_t* ent_off, const void* kv, const int64_t* kv_off,
                            const int64_t* kv_pos0, const int32_t* q_seq, const int32_t* q_pos,
                            int32_t m, const float* sink, int32_t Q, int32_t B, int32_t H,
                            int32_t D, int32_t W, float softmax_scale, float rope_theta,
                            float eps, int32_t max_n, void* out, void* workspace,
                            size_t workspace_bytes, const csa_cache_layout_t* layout,
                            int32_t* dev_status, void* stream) {
    REQUIRE(Q >= 0, "Q must be >= 0");
    if (Q == 0) return ok();
    csa_status_t v = attn_validate(q, entries, fmt, ent_rows, seq_len, ent_off, kv, kv_off, kv_pos0, q_seq, q_pos,
                                   sink, B, H, D, W, m, softmax_scale, rope_theta, eps, out);
    if (v != CSA_OK) return v;
    REQUIRE(max_n >= 0, "max_n must be >= 0");
    const size_t need = dense_hca_workspace_size(Q, H, D, max_n);
    if (!workspace || workspace_bytes < need || !aligned(workspace, 256))
        return fail(CSA_ERR_WORKSPACE, "workspace must be >= %zu bytes, 256-byte aligned", need);
    SUPPORT(!layout || !layout->block_table,
            "dense attention reads contiguous entries: no block table");
    csa::EntryRows er;
    csa::RawRows raw;
    v = make_rows(layout, m, ent_off, kv_off, kv_pos0, true, &er, &raw);
    if (v != CSA_OK) return v;
    csa::AttnArgs a{(const uint16_t*)q, (const uint8_t*)entries, er, (const uint16_t*)kv,
                    raw, q_seq, q_pos, seq_len, nullptr, ent_rows, sink, (uint16_t*)out, dev_status,
                    0, m, B, H, W, fmt, softmax_scale, eps, log2((double)rope_theta)};
    if (csa::attn_tc_supported(H, D, fmt))
        return cuda_status(csa::launch_attn_tc(a, Q, max_n, workspace, (cudaStream_t)stream),
                           "attention launch");
    return cuda_status(csa::launch_attn_simt(a, Q, D, (cudaStream_t)stream), "attention launch");
}

}  // extern "C"
