// Internal launcher declarations shared by the kernel files and the C ABI layer.
#pragma once

#include "common.cuh"

#include <utility>

namespace csa {

// Launches `kernel` with programmatic stream serialization allowed (see pdl_wait).
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// As launch_pdl, in thread-block clusters of `cluster_x` CTAs along x.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl_cluster(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                               cudaStream_t stream, int cluster_x, Args&&... args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    attr[1].id = cudaLaunchAttributeClusterDimension;
    attr[1].val.clusterDim.x = (unsigned)cluster_x;
    attr[1].val.clusterDim.y = 1;
    attr[1].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Kernel kinds for launch accounting (names in prof.cu).
enum KernelKind {
    kKCompress = 0,
    kKTopk,
    kKAttnSimt,
    kKIndexerTc,
    kKAttnTc,
    kKAttnCombine,
    kKAttn576Tc,
    kKTopkMerge,
    kKCpCandidates,
    kKCpPackRows,
    kKIndexerFp4,
    kKCacheAppend,
    kKernelKinds
};

// Counts one kernel launch; with timing enabled, brackets it with CUDA events on `stream`.
class LaunchScope {
  public:
    LaunchScope(int kind, cudaStream_t stream);
    ~LaunchScope();
    LaunchScope(const LaunchScope&) = delete;
    LaunchScope& operator=(const LaunchScope&) = delete;

  private:
    int kind_;
    cudaStream_t stream_;
    cudaEvent_t start_ = nullptr, stop_ = nullptr;
};

struct AttnArgs {
    const uint16_t* q;
    const uint8_t* entries;
    EntryRows er;        // where the classical cache holds entry i of sequence b
    const uint16_t* kv;
    RawRows raw;         // where the state cache holds raw token p of sequence b
    const int32_t* q_seq;
    const int32_t* q_pos;
    const int64_t* seq_len;
    const int32_t* idx;  // nullptr = dense over all visible entries
    int64_t ent_rows;
    const float* sink;
    uint16_t* out;
    int32_t* st;
    int k, m, B, H, W, fmt;
    float scale, eps;
    double log2_theta;
};

cudaError_t launch_compress(int span, const void* kv, const void* gate, const float* bias,
                            const int64_t* seq_len, const RawRows& raw, const EntryRows& er,
                            const int32_t* item_seq, const int32_t* item_ent, int64_t n_items,
                            int B, int m, int D, int fmt, float theta, float eps, void* entries,
                            int32_t* st, cudaStream_t stream);
bool indexer_tc_supported(int HI, int dI);
cudaError_t launch_indexer_tc(const uint8_t* qI, const float* qs, const float* w,
                              const uint8_t* kI, const float* ks, int64_t ent_rows,
                              const int64_t* seq_len, const EntryRows& er,
                              const int32_t* q_seq, const int32_t* q_pos, int Q, int B, int HI,
                              int dI, int m, int max_n, float* scores, int64_t ld, int32_t* st,
                              cudaStream_t stream, uint32_t* gmax = nullptr, int64_t ld_g = 0);
bool indexer_fp4_supported(int HI, int dI);
cudaError_t launch_indexer_fp4(const uint8_t* qI, const uint8_t* qI_sf, const float* w,
                               const uint8_t* kI, const uint8_t* kI_sf, int64_t ent_rows,
                               const int64_t* seq_len, const EntryRows& er,
                               const int32_t* q_seq, const int32_t* q_pos, int Q, int B, int HI,
                               int m, int max_n, int bf16, float* scores, int64_t ld,
                               int32_t* st, cudaStream_t stream, uint32_t* gmax, int64_t ld_g);
cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_seq,
                        const int32_t* q_pos, const int64_t* seq_len, int Q, int B, int m,
                        int max_n, int k, int32_t* idx_out, int32_t* st, cudaStream_t stream,
                        const uint32_t* gmax = nullptr, int64_t ld_g = 0);
cudaError_t launch_attn_simt(const AttnArgs& a, int Q, int D, cudaStream_t stream);
bool attn_tc_supported(int H, int D, int fmt);
bool attn576_tc_supported(int H, int D, int fmt);
cudaError_t launch_attn576_tc(const AttnArgs& a, int Q, cudaStream_t stream);
size_t attn_tc_workspace_bytes(int Q, int max_n);
cudaError_t launch_attn_tc(const AttnArgs& a, int Q, int max_n, void* workspace,
                           cudaStream_t stream);

bool topk_merge_supported(int n_cand, int k);
cudaError_t launch_topk_merge(const float* cand_scores, const int32_t* cand_idx,
                              int64_t slice_stride, int W, int Q, int k_in, int k,
                              int32_t* idx_out, int32_t* st, cudaStream_t stream);
cudaError_t launch_cp_candidates(const int32_t* idx, const float* scores, int64_t ld,
                                 const int32_t* q_seq, const int64_t* lo, int Q, int B, int k,
                                 int32_t* cand_idx, float* cand_scores, int32_t* st,
                                 cudaStream_t stream);
cudaError_t launch_cp_pack_rows(const int32_t* idx, const int32_t* q_seq, const int64_t* lo,
                                const int64_t* n, const int64_t* ent_off,
                                const uint8_t* entries, int64_t ent_rows, int row_bytes, int Q,
                                int B, int k, uint8_t* out, int32_t* local_idx, int32_t* st,
                                cudaStream_t stream);

cudaError_t launch_cache_append(const uint16_t* kv_new, const uint16_t* gate_new,
                                const uint8_t* kI_new, const float* ks_new, int64_t* seq_len,
                                const RawRows& raw, const EntryRows& er, int B, int D, int dI,
                                int m, int64_t kv_rows, int64_t ent_rows, uint16_t* kv,
                                uint16_t* gate, uint8_t* kI, float* ks, int32_t* st,
                                cudaStream_t stream);

// Sets the thread-local message csa_last_error() returns (printf-style).
void set_error_message(const char* fmt, ...);

}  // namespace csa
