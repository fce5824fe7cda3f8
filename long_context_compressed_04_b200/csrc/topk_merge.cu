// Top-k merge for context-parallel decode (the plan of the stuffyNLP post's context
// parallelism, applied to the selection of "DeepSeek-V4 深度分析报告" 2.1 CSA).
//
// A sequence's compressed entries are split into contiguous slices, one per rank; each
// rank selects the top-k of its slice with lightning_indexer_topk.  Every entry of the
// sequence's top-k is in its slice's top-k (the order within a slice is the order of the
// whole sequence), so the sequence's top-k is the top-k of the union of the slices'.  This
// kernel takes, per query, the candidates -- each slice's index set (global entry indices,
// ascending) and scores, slices in rank order, so the candidates are in ascending global
// order -- and selects k of them under the order of the selection: larger score first,
// lower entry index first among equal scores (-0 = +0).  It writes them in ascending entry
// order, -1 padded, exactly as lightning_indexer_topk over the whole sequence would.
//
// One CTA of 1024 threads per query.  The k-th largest key T and the number krem of keys
// equal to T to take are found by 11-bit radix digits over the candidates in shared memory;
// then each candidate is taken if its key is > T, or == T and fewer than krem ties precede
// it, and one scan places the taken ones.
#include "launchers.cuh"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kPer = 16;                       // candidates per thread
constexpr int kMaxCand = kThreads * kPer;      // 16384: e.g. 8 ranks x k = 2048

struct MergeShared {
    uint32_t key[kMaxCand];
    uint32_t hist[kBins];
    uint32_t scan[kWarps + 1];
    uint32_t or_and[2];
    uint32_t bin, krem;
};

// Exclusive prefix sum of `v` over the CTA; `total` gets the sum.  Ends synchronised.
__device__ __forceinline__ uint32_t cta_exclusive_scan(uint32_t v, uint32_t* tmp, uint32_t& total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    uint32_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) tmp[wid] = x;
    __syncthreads();
    if (wid == 0) {
        const uint32_t w = lane < kWarps ? tmp[lane] : 0u;
        uint32_t inc = w;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        __syncwarp();
        tmp[lane] = inc - w;
        if (lane == 31) tmp[kWarps] = inc;
    }
    __syncthreads();
    const uint32_t res = x - v + tmp[wid];
    total = tmp[kWarps];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(kThreads) topk_merge_kernel(
    const float* __restrict__ cand_scores, const int32_t* __restrict__ cand_idx, int n_cand,
    int k, int32_t* __restrict__ idx_out, int32_t* __restrict__ dev_status) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    MergeShared& sh = *reinterpret_cast<MergeShared*>(smem_raw);
    const int q = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const float* s = cand_scores + (int64_t)q * n_cand;
    const int32_t* ix = cand_idx + (int64_t)q * n_cand;
    int32_t* out = idx_out + (int64_t)q * k;
    // the candidates come from the selections before this kernel; the output may still be
    // read by the kernel before it
    pdl_wait();
    pdl_trigger();
    // my candidates: a contiguous run of kPer, in order; key 0 marks a pad (every score's
    // key is > 0 except that of a -NaN, flagged below)
    const int c0 = tid * kPer;
    uint32_t valid = 0u;   // bit j: candidate c0 + j is an entry
    uint32_t kor = 0u, kand = 0xFFFFFFFFu, nval = 0u;
#pragma unroll
    for (int j = 0; j < kPer; j++) {
        const int c = c0 + j;
        uint32_t key = 0u;
        if (c < n_cand && ix[c] >= 0) {
            const float v = s[c];
            if (v != v) flag(dev_status, CSA_DEV_NAN);
            key = order_key(v);
            valid |= 1u << j;
            kor |= key;
            kand &= key;
            nval++;
        }
        sh.key[c] = key;
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kor |= __shfl_xor_sync(0xffffffffu, kor, o);
        kand &= __shfl_xor_sync(0xffffffffu, kand, o);
    }
    if (tid == 0) {
        sh.or_and[0] = 0u;
        sh.or_and[1] = 0xFFFFFFFFu;
    }
    __syncthreads();
    if (lane == 0) {
        atomicOr(&sh.or_and[0], kor);
        atomicAnd(&sh.or_and[1], kand);
    }
    uint32_t total;
    const uint32_t before = cta_exclusive_scan(nval, sh.scan, total);
    if (total <= (uint32_t)k) {
        // every candidate is taken (at most k visible entries), in order, then -1
        uint32_t pos = before;
#pragma unroll
        for (int j = 0; j < kPer; j++)
            if ((valid >> j) & 1u) out[pos++] = ix[c0 + j];
        for (int j = (int)total + tid; j < k; j += kThreads) out[j] = -1;
        return;
    }
    // T, the k-th largest key, and krem, how many keys equal to T are taken
    const uint32_t vary = sh.or_and[0] ^ sh.or_and[1];
    uint32_t prefix = sh.or_and[1] & ~vary, mask = ~vary, krem = (uint32_t)k;
    int top = vary ? 31 - __clz(vary) : -1;
    while (top >= 0) {
        const int width = top >= 10 ? 11 : top + 1;
        const int shift = top + 1 - width;
        const uint32_t bmask = (1u << width) - 1u;
        for (int x = tid; x < kBins; x += kThreads) sh.hist[x] = 0u;
        __syncthreads();
#pragma unroll
        for (int j = 0; j < kPer; j++) {
            const uint32_t key = sh.key[c0 + j];
            if (((valid >> j) & 1u) && (key & mask) == prefix)
                atomicAdd(&sh.hist[(key >> shift) & bmask], 1u);
        }
        __syncthreads();
        // bins scanned from the top: 2 per thread
        const int bhi = kBins - 1 - 2 * tid, blo = bhi - 1;
        const uint32_t chi = sh.hist[bhi], clo = sh.hist[blo];
        uint32_t tot2;
        const uint32_t above = cta_exclusive_scan(chi + clo, sh.scan, tot2);
        if (above < krem && krem <= above + chi) {
            sh.bin = (uint32_t)bhi;
            sh.krem = krem - above;
        } else if (above + chi < krem && krem <= above + chi + clo) {
            sh.bin = (uint32_t)blo;
            sh.krem = krem - above - chi;
        }
        __syncthreads();
        krem = sh.krem;
        prefix |= sh.bin << shift;
        mask |= bmask << shift;
        top = shift - 1;
        __syncthreads();
    }
    const uint32_t T = prefix;
    // taken: key > T, or key == T with fewer than krem ties before it (in candidate order,
    // which is ascending entry order)
    uint32_t nt = 0u;
#pragma unroll
    for (int j = 0; j < kPer; j++)
        if (((valid >> j) & 1u) && sh.key[c0 + j] == T) nt++;
    uint32_t t3;
    uint32_t ties = cta_exclusive_scan(nt, sh.scan, t3);
    uint32_t take = 0u;
#pragma unroll
    for (int j = 0; j < kPer; j++) {
        if (!((valid >> j) & 1u)) continue;
        const uint32_t key = sh.key[c0 + j];
        if (key > T) {
            take |= 1u << j;
        } else if (key == T) {
            if (ties < krem) take |= 1u << j;
            ties++;
        }
    }
    uint32_t t4;
    uint32_t pos = cta_exclusive_scan((uint32_t)__popc(take), sh.scan, t4);
#pragma unroll
    for (int j = 0; j < kPer; j++)
        if ((take >> j) & 1u) {
            if (pos < (uint32_t)k) out[pos] = ix[c0 + j];
            pos++;
        }
    if (tid == 0 && t4 != (uint32_t)k) flag(dev_status, CSA_DEV_NAN);   // no total order
}

}  // namespace

bool topk_merge_supported(int n_cand, int k) { return n_cand >= 1 && n_cand <= kMaxCand && k >= 1; }

cudaError_t launch_topk_merge(const float* cand_scores, const int32_t* cand_idx, int Q,
                              int n_cand, int k, int32_t* idx_out, int32_t* st,
                              cudaStream_t stream) {
    if (Q == 0) return cudaSuccess;
    const size_t smem = sizeof(MergeShared);
    cudaError_t e = cudaFuncSetAttribute(topk_merge_kernel,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    LaunchScope scope(kKTopkMerge, stream);
    return launch_pdl(topk_merge_kernel, dim3(Q), dim3(kThreads), smem, stream, cand_scores,
                      cand_idx, n_cand, k, idx_out, st);
}

}  // namespace csa
