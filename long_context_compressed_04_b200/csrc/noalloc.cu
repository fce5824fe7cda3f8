// lightning_indexer_topk_noalloc: the lightning indexer + top-k for callers that cannot
// allocate device memory.
//
// Some callers of this library cannot call cudaMalloc or hand it a workspace: a plugin
// running inside a host framework that owns every byte of the device memory pool and
// gives its plugins no scratch, or a latency-critical serving loop in which a cudaMalloc
// (which can synchronise the device) is not allowed.  This entry point takes the same
// inputs and outputs as lightning_indexer_topk but keeps its scratch -- the per-query
// score rows the selection reads -- in one statically sized device array that lives in
// this library's module.  It calls the existing lightning_indexer_topk with that array
// as the workspace, so the results are the same.
//
// Limits and caveats (also stated in include/csa.h):
//  - the array holds CSA_NOALLOC_SCRATCH_BYTES bytes; a call whose
//    csa_indexer_workspace_size(Q, max_n, k) is larger fails with CSA_ERR_WORKSPACE and
//    launches nothing;
//  - every GPU that loads the library keeps the array until the process exits;
//  - all calls on a device share the one array and it keeps what the last call wrote;
//    nothing in it needs to start at zero (each score is written before it is read), but
//    calls whose kernels overlap on the GPU (different streams, no ordering) race on it;
//  - with scores_out given, the scores go there and the array is not used (no size limit);
//  - each call that is not being captured into a CUDA graph looks up the array's device
//    address with cudaGetSymbolAddress on the current device and caches it; a call made
//    during stream capture uses the cached address, so make one call on each device before
//    capturing (and again after a cudaDeviceReset, which invalidates the cached address).
#include <mutex>

#include "launchers.cuh"

namespace {

static __device__ __align__(256) unsigned char g_indexer_scratch[CSA_NOALLOC_SCRATCH_BYTES];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

extern "C" csa_status_t lightning_indexer_topk_noalloc(
    const uint8_t* qI, const float* qI_scale, const float* w, const uint8_t* kI,
    const float* kI_scale, int64_t ent_rows, const int64_t* seq_len, const int64_t* ent_off, const int32_t* q_seq,
    const int32_t* q_pos, int32_t Q, int32_t B, int32_t H_I, int32_t d_I, int32_t m, int32_t k,
    int32_t max_n, int32_t* idx_out, float* scores_out, int64_t ld_scores, int32_t* dev_status,
    void* stream) {
    // the scores go to the caller's buffer (no scratch needed), or there is nothing to do,
    // or the arguments are invalid: lightning_indexer_topk handles and reports these
    const size_t need = csa_indexer_workspace_size(Q, max_n, k);
    if (Q <= 0 || scores_out != nullptr || need == 0)
        return lightning_indexer_topk(qI, qI_scale, w, kI, kI_scale, ent_rows, seq_len, ent_off,
                                      q_seq, q_pos, Q, B, H_I, d_I, m, k, max_n, idx_out,
                                      scores_out, ld_scores, nullptr, 0, nullptr, dev_status,
                                      stream);
    if (need > (size_t)CSA_NOALLOC_SCRATCH_BYTES) {
        csa::set_error_message("lightning_indexer_topk_noalloc: Q=%d, max_n=%d needs %zu bytes of "
                              "scratch, more than the built-in %zu",
                              Q, max_n, need, (size_t)CSA_NOALLOC_SCRATCH_BYTES);
        return CSA_ERR_WORKSPACE;
    }
    int dev = -1;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
        csa::set_error_message("lightning_indexer_topk_noalloc: no usable current device (%s)",
                              cudaGetErrorString(e));
        return CSA_ERR_CUDA;
    }
    cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
    if (cudaStreamIsCapturing((cudaStream_t)stream, &cap) != cudaSuccess) {
        csa::set_error_message("lightning_indexer_topk_noalloc: invalid stream");
        return CSA_ERR_INVALID_ARG;
    }
    void* scratch = nullptr;
    {
        std::lock_guard<std::mutex> lk(g_mu);
        if (cap == cudaStreamCaptureStatusNone || !g_scratch_ptr[dev]) {
            void* p = nullptr;
            e = cudaGetSymbolAddress(&p, g_indexer_scratch);
            if (e != cudaSuccess || p == nullptr) {
                csa::set_error_message(
                    "lightning_indexer_topk_noalloc: cudaGetSymbolAddress failed on device %d: %s",
                    dev, cudaGetErrorString(e));
                return CSA_ERR_CUDA;
            }
            g_scratch_ptr[dev] = p;
        }
        scratch = g_scratch_ptr[dev];
    }
    return lightning_indexer_topk(qI, qI_scale, w, kI, kI_scale, ent_rows, seq_len, ent_off, q_seq, q_pos,
                                  Q, B, H_I, d_I, m, k, max_n, idx_out, scores_out, ld_scores,
                                  scratch, (size_t)CSA_NOALLOC_SCRATCH_BYTES, nullptr, dev_status,
                                  stream);
}
