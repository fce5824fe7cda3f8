// Step a4: per-query top-k over the indexer scores.
//
// "DeepSeek-V4 深度分析报告" 2.1 CSA: keep the k best compressed entries per query
// (k = 512 / 1024).  The selection order is total: larger score first, lower entry index
// first among equal scores (-0 and +0 are equal), so the selected set is unique and does
// not depend on how the work is partitioned -- the result is batch-invariant by
// construction.
//
// One CTA (1024 threads) per query: a 4-pass radix select (8 bits per pass) over
// order-preserving 32-bit keys finds the k-th largest key T and how many of the keys equal
// to T are needed; a final pass in ascending entry order takes every key > T and the first
// needed keys == T, writing them with a block-wide prefix sum -- which emits the indices
// already in ascending order.
#include "launchers.cuh"

namespace csa {

__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;  // -0 ties with +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the CTA; `total` receives the CTA sum.  tmp holds >= 33 ints.
__device__ __forceinline__ int block_exclusive_scan(int v, int* tmp, int& total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    const int nw = blockDim.x >> 5;
    int x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) tmp[wid] = x;
    __syncthreads();
    if (wid == 0) {
        const int wv = lane < nw ? tmp[lane] : 0;
        int inc = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        __syncwarp();
        tmp[lane] = inc - wv;
        if (lane == 31) tmp[32] = inc;
    }
    __syncthreads();
    const int res = x - v + tmp[wid];
    total = tmp[32];
    __syncthreads();
    return res;
}

__global__ void __launch_bounds__(1024) topk_radix_kernel(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ q_seq,
    const int32_t* __restrict__ q_pos, const int64_t* __restrict__ seq_len, int B, int m,
    int max_n, int k, int32_t* __restrict__ idx_out, int32_t* __restrict__ dev_status) {
    __shared__ uint32_t hist[256];
    __shared__ int scan_tmp[2][33];
    __shared__ uint32_t sh_prefix;
    __shared__ int sh_krem;
    const int qq = blockIdx.x;
    const int tid = threadIdx.x;
    const int b = q_seq[qq];
    const int t = q_pos[qq];
    // invalid queries (flagged by the scoring kernel) select nothing
    const bool valid = b >= 0 && b < B && t >= 0 && (int64_t)t < seq_len[b];
    int n = valid ? (t + 1) / m : 0;
    if (n > max_n) n = max_n;  // capacity already flagged by the scoring kernel
    const float* s = scores + (int64_t)qq * ld;
    int32_t* out = idx_out + (int64_t)qq * k;
    if (n <= k) {
        for (int j = tid; j < k; j += blockDim.x) out[j] = j < n ? j : -1;
        return;
    }
    uint32_t prefix = 0u, mask = 0u;
    int krem = k;
    for (int shift = 24; shift >= 0; shift -= 8) {
        for (int x = tid; x < 256; x += blockDim.x) hist[x] = 0u;
        __syncthreads();
        for (int i = tid; i < n; i += blockDim.x) {
            const uint32_t key = score_key(s[i]);
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
        }
        __syncthreads();
        if (tid == 0) {
            int cum = 0;
            for (int bin = 255; bin >= 0; bin--) {
                const int h = (int)hist[bin];
                if (cum + h >= krem) {
                    sh_prefix = prefix | ((uint32_t)bin << shift);
                    sh_krem = krem - cum;
                    break;
                }
                cum += h;
            }
        }
        __syncthreads();
        prefix = sh_prefix;
        krem = sh_krem;
        mask |= 255u << shift;
        __syncthreads();
    }
    const uint32_t T = prefix;  // the k-th largest key; krem keys equal to T are needed
    int written = 0, ties_seen = 0;
    for (int i0 = 0; i0 < n; i0 += blockDim.x) {
        const int i = i0 + tid;
        const uint32_t key = i < n ? score_key(s[i]) : 0u;
        const int gt = (i < n) && key > T;
        const int eq = (i < n) && key == T;
        int eq_total, sel_total;
        const int eq_rank = block_exclusive_scan(eq, scan_tmp[0], eq_total);
        const int sel = gt || (eq && ties_seen + eq_rank < krem);
        const int pos = block_exclusive_scan(sel, scan_tmp[1], sel_total);
        if (sel && written + pos < k) out[written + pos] = i;
        written += sel_total;
        ties_seen += eq_total;
    }
    if (tid == 0 && written != k) flag(dev_status, CSA_DEV_NAN);  // only NaN keys can do this
}

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_seq,
                        const int32_t* q_pos, const int64_t* seq_len, int Q, int B, int m,
                        int max_n, int k, int32_t* idx_out, int32_t* st, cudaStream_t stream) {
    if (Q == 0) return cudaSuccess;
    LaunchScope scope(kKTopk, stream);
    topk_radix_kernel<<<Q, 1024, 0, stream>>>(scores, ld, q_seq, q_pos, seq_len, B, m, max_n, k,
                                              idx_out, st);
    return cudaGetLastError();
}

}  // namespace csa
