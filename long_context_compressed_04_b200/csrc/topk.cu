// Step a4: per-query top-k over the indexer scores.
//
// "DeepSeek-V4 深度分析报告" 2.1 CSA: keep the k best compressed entries per query
// (k = 512 / 1024).  The selection order is total: larger score first, lower entry index
// first among equal scores (-0 and +0 are equal), so the selected set is unique and does
// not depend on how the work is partitioned -- the result is batch-invariant by
// construction.
//
// One CTA (1024 threads) per query.  Scores map to order-preserving 32-bit keys.  Three
// radix passes (11, 11 and 10 bits) find the k-th largest key T and how many keys equal
// to T are needed: each pass histograms the keys that match the prefix found so far with
// warp-aggregated shared-memory atomics (lanes hitting the same bin add once), then a
// block-wide scan over the 2048 bins, from the top, picks the bin holding the k-th key.
// A last pass in ascending entry order takes every key > T and the first needed keys
// == T; one block-wide scan per 4096-entry chunk gives each thread its output slots, so
// the indices come out already sorted.  Score rows are read with 16-byte loads.
#include "launchers.cuh"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kChunk = 4 * kThreads;

__device__ __forceinline__ uint32_t score_key(float s) {
    uint32_t u = __float_as_uint(s);
    if (u == 0x80000000u) u = 0u;  // -0 ties with +0
    return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive prefix sum over the CTA of `v`; `total` gets the CTA sum.  tmp: >= 33 ints.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* tmp,
                                                         uint32_t& total) {
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
        const uint32_t wv = lane < kWarps ? tmp[lane] : 0u;
        uint32_t inc = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        __syncwarp();
        tmp[lane] = inc - wv;
        if (lane == 31) tmp[32] = inc;
    }
    __syncthreads();
    const uint32_t res = x - v + tmp[wid];
    total = tmp[32];
    __syncthreads();
    return res;
}

// Keys of entries i .. i+3 (0 past n).  `vec`: the row is 16-byte aligned.
__device__ __forceinline__ void load4(const float* s, int i, int n, bool vec, uint32_t* key) {
    if (vec && i + 3 < n) {
        const float4 v = *reinterpret_cast<const float4*>(s + i);
        key[0] = score_key(v.x);
        key[1] = score_key(v.y);
        key[2] = score_key(v.z);
        key[3] = score_key(v.w);
    } else {
#pragma unroll
        for (int u = 0; u < 4; u++) key[u] = (i + u < n) ? score_key(s[i + u]) : 0u;
    }
}

__global__ void __launch_bounds__(kThreads) topk_radix_kernel(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ q_seq,
    const int32_t* __restrict__ q_pos, const int64_t* __restrict__ seq_len, int B, int m,
    int max_n, int k, int32_t* __restrict__ idx_out, int32_t* __restrict__ dev_status) {
    __shared__ uint32_t hist[kBins];
    __shared__ uint32_t scan_tmp[33];
    __shared__ uint32_t sh_bin, sh_krem;
    const int qq = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31;
    const int b = q_seq[qq];
    const int t = q_pos[qq];
    // invalid queries (flagged by the scoring kernel) select nothing
    const bool valid = b >= 0 && b < B && t >= 0 && (int64_t)t < seq_len[b];
    int n = valid ? (t + 1) / m : 0;
    if (n > max_n) n = max_n;  // capacity already flagged by the scoring kernel
    const float* s = scores + (int64_t)qq * ld;
    int32_t* out = idx_out + (int64_t)qq * k;
    if (n <= k) {
        for (int j = tid; j < k; j += kThreads) out[j] = j < n ? j : -1;
        return;
    }
    const bool vec = (reinterpret_cast<uintptr_t>(s) & 15) == 0;

    uint32_t prefix = 0u, mask = 0u, krem = (uint32_t)k;
    for (int pass = 0; pass < 3; pass++) {
        const int shift = pass == 0 ? 21 : (pass == 1 ? 10 : 0);
        const uint32_t bmask = pass == 2 ? 1023u : 2047u;
        for (int x = tid; x < kBins; x += kThreads) hist[x] = 0u;
        __syncthreads();
        for (int c0 = 0; c0 < n; c0 += kChunk) {   // uniform trip count: whole warps
            const int i0 = c0 + 4 * tid;
            uint32_t key[4];
            load4(s, i0, n, vec, key);
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const bool hit = (i0 + u < n) && ((key[u] & mask) == prefix);
                const uint32_t bin = hit ? ((key[u] >> shift) & bmask) : 0xFFFFFFFFu;
                const uint32_t peers = __match_any_sync(0xffffffffu, bin);
                if (hit && lane == __ffs(peers) - 1) atomicAdd(&hist[bin], (uint32_t)__popc(peers));
            }
        }
        __syncthreads();
        // bins from the top: thread t owns bins 2047 - 2t and 2046 - 2t
        const int bhi = kBins - 1 - 2 * tid, blo = bhi - 1;
        const uint32_t chi = hist[bhi], clo = hist[blo];
        uint32_t tot;
        const uint32_t above = block_exclusive_scan(chi + clo, scan_tmp, tot);
        if (above < krem && krem <= above + chi) {
            sh_bin = (uint32_t)bhi;
            sh_krem = krem - above;
        } else if (above + chi < krem && krem <= above + chi + clo) {
            sh_bin = (uint32_t)blo;
            sh_krem = krem - above - chi;
        }
        __syncthreads();
        prefix |= sh_bin << shift;
        mask |= bmask << shift;
        krem = sh_krem;
        __syncthreads();
    }
    const uint32_t T = prefix;   // the k-th largest key; krem keys equal to T are taken
    // ordered collection: 4096 entries per round, 4 consecutive per thread
    uint32_t written = 0, ties_before = 0;
    for (int c0 = 0; c0 < n; c0 += kChunk) {
        const int i0 = c0 + 4 * tid;
        uint32_t key[4];
        load4(s, i0, n, vec, key);
        uint32_t ngt = 0, neq = 0;
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const bool in = i0 + u < n;
            ngt += (in && key[u] > T) ? 1u : 0u;
            neq += (in && key[u] == T) ? 1u : 0u;
        }
        uint32_t tot;
        const uint32_t packed = block_exclusive_scan(ngt | (neq << 16), scan_tmp, tot);
        uint32_t eq_rank = ties_before + (packed >> 16);   // tie rank of my first tie
        uint32_t pos = written + (packed & 0xFFFFu) + (min(eq_rank, krem) - min(ties_before, krem));
#pragma unroll
        for (int u = 0; u < 4; u++) {
            const bool in = i0 + u < n;
            bool take = in && key[u] > T;
            if (in && key[u] == T) {
                take = eq_rank < krem;
                eq_rank++;
            }
            if (take) {
                if (pos < (uint32_t)k) out[pos] = i0 + u;
                pos++;
            }
        }
        const uint32_t ties_after = ties_before + (tot >> 16);
        written += (tot & 0xFFFFu) + (min(ties_after, krem) - min(ties_before, krem));
        ties_before = ties_after;
    }
    if (tid == 0 && written != (uint32_t)k) flag(dev_status, CSA_DEV_NAN);
}

}  // namespace

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_seq,
                        const int32_t* q_pos, const int64_t* seq_len, int Q, int B, int m,
                        int max_n, int k, int32_t* idx_out, int32_t* st, cudaStream_t stream) {
    if (Q == 0) return cudaSuccess;
    LaunchScope scope(kKTopk, stream);
    topk_radix_kernel<<<Q, kThreads, 0, stream>>>(scores, ld, q_seq, q_pos, seq_len, B, m, max_n,
                                                  k, idx_out, st);
    return cudaGetLastError();
}

}  // namespace csa
