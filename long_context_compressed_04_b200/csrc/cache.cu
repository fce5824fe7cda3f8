// Appending one decode token per sequence to the hybrid cache ("DeepSeek-V4 深度分析报告"
// 3.5, KV cache management: the state cache keeps the sliding-window KV and the tokens not
// yet compressed; the classical cache keeps the compressed entries in blocks of 128 tokens).
//
// One CTA per sequence: the new token's raw KV and gate rows go to its state-cache row
// (ring slot p mod kv_ring, or the linear row), and when the token completes a block of m
// the new entry's indexer key row and scale go to the entry's row of the key store (through
// the block table when there is one); then seq_len[b] becomes p + 1.  The compression of the
// new entry itself is a csa_compress call after this one.
//
// The kernel never lets the next kernel start early (no launch_dependents): the next
// kernels read seq_len and the raw rows before their own wait on this grid.
#include "launchers.cuh"

namespace csa {

namespace {

__global__ void __launch_bounds__(128) cache_append_kernel(
    const uint16_t* __restrict__ kv_new, const uint16_t* __restrict__ gate_new,
    const uint8_t* __restrict__ kI_new, const float* __restrict__ ks_new, int64_t* seq_len,
    RawRows raw, EntryRows er, int B, int D, int dI, int m, int64_t kv_rows, int64_t ent_rows,
    uint16_t* __restrict__ kv, uint16_t* __restrict__ gate, uint8_t* __restrict__ kI,
    float* __restrict__ ks, int32_t* __restrict__ st) {
    const int b = blockIdx.x;
    // the previous step's kernels may still read the rows and seq_len written here
    pdl_wait();
    const int64_t p = seq_len[b];
    const int64_t row = raw.row(b, p);
    if (row < 0 || row >= kv_rows) {
        if (threadIdx.x == 0) flag(st, CSA_DEV_OOB);
        return;
    }
    const int n16 = D * 2 / 16;
    const uint4* src_k = reinterpret_cast<const uint4*>(kv_new + (int64_t)b * D);
    const uint4* src_g = reinterpret_cast<const uint4*>(gate_new + (int64_t)b * D);
    uint4* dst_k = reinterpret_cast<uint4*>(kv + row * D);
    uint4* dst_g = reinterpret_cast<uint4*>(gate + row * D);
    for (int c = threadIdx.x; c < n16; c += blockDim.x) {
        dst_k[c] = src_k[c];
        dst_g[c] = src_g[c];
    }
    bool ok = true;
    if (kI_new && (p + 1) % m == 0) {
        const int64_t e = (p + 1) / m - 1;
        const int64_t erow = er.row(b, e);
        if (erow < 0 || erow >= ent_rows) {
            if (threadIdx.x == 0) flag(st, CSA_DEV_OOB);
            ok = false;
        } else {
            const uint4* sk = reinterpret_cast<const uint4*>(kI_new + (int64_t)b * dI);
            uint4* dk = reinterpret_cast<uint4*>(kI + erow * dI);
            for (int c = threadIdx.x; c < dI / 16; c += blockDim.x) dk[c] = sk[c];
            if (threadIdx.x == 0) ks[erow] = ks_new[b];
        }
    }
    __syncthreads();
    if (threadIdx.x == 0 && ok) seq_len[b] = p + 1;
}

}  // namespace

cudaError_t launch_cache_append(const uint16_t* kv_new, const uint16_t* gate_new,
                                const uint8_t* kI_new, const float* ks_new, int64_t* seq_len,
                                const RawRows& raw, const EntryRows& er, int B, int D, int dI,
                                int m, int64_t kv_rows, int64_t ent_rows, uint16_t* kv,
                                uint16_t* gate, uint8_t* kI, float* ks, int32_t* st,
                                cudaStream_t stream) {
    if (B == 0) return cudaSuccess;
    LaunchScope scope(kKCacheAppend, stream);
    return launch_pdl(cache_append_kernel, dim3(B), dim3(128), 0, stream, kv_new, gate_new,
                      kI_new, ks_new, seq_len, raw, er, B, D, dI, m, kv_rows, ent_rows, kv, gate,
                      kI, ks, st);
}

}  // namespace csa
