// Context-parallel decode (the plan of the stuffyNLP post's context parallelism, applied to
// the selection and attention of "DeepSeek-V4 深度分析报告" 2.1 CSA).
//
// A sequence's compressed entries are split into contiguous slices, one per rank; each
// rank selects the top-k of its slice with lightning_indexer_topk.  Every entry of the
// sequence's top-k is in its slice's top-k (the order within a slice is the order of the
// whole sequence), so the sequence's top-k is the top-k of the union of the slices'.
//
//  - cp_candidates_kernel turns a slice's selection (slice-local indices, -1 padded) and its
//    score rows into candidates: entry indices of the whole sequence and their scores.
//  - topk_merge_kernel takes, per query, the W slices' candidates (slice-major, slices in
//    ascending entry order, so the candidates are in ascending entry order) and selects k
//    of them under the order of the selection: larger score first, lower entry index first
//    among equal scores (-0 = +0).  It writes them in ascending entry order, -1 padded,
//    exactly as lightning_indexer_topk over the whole sequence would.  One CTA of 1024
//    threads per query, 4, 8 or 16 consecutive candidates in each thread's registers: the k-th
//    largest key T and the number krem of keys equal to T to take are found by 11-bit
//    radix digits (histograms in shared memory); then each
//    candidate is taken if its key is > T, or == T and fewer than krem ties precede it, and
//    one scan places the taken ones.
//  - cp_pack_rows_kernel writes, at each selected position, the entry row if this rank's
//    slice holds it and zeros otherwise: every position has exactly one rank with a
//    non-zero row, so an integer sum over the ranks' buffers is the gather of the rows.
//    It also writes the selection renumbered to those positions (j, or -1), which is what
//    the attention reads the gathered rows with.
#include "launchers.cuh"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kMaxCand = kThreads * 16;        // 16384: e.g. 8 ranks x k = 2048

struct MergeShared {
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

// Candidate c = r * k_in + j of query q (slice r, position j) is element
// r * slice_stride + q * k_in + j of cand_scores / cand_idx.
// PER candidates per thread (kThreads * PER >= n_cand).
template <int PER>
__global__ void __launch_bounds__(kThreads, 1) topk_merge_kernel(
    const float* __restrict__ cand_scores, const int32_t* __restrict__ cand_idx,
    int64_t slice_stride, int k_in, int n_cand, int k, int32_t* __restrict__ idx_out,
    int32_t* __restrict__ dev_status) {
    extern __shared__ __align__(16) uint8_t smem_raw[];
    MergeShared& sh = *reinterpret_cast<MergeShared*>(smem_raw);
    const int q = blockIdx.x, tid = threadIdx.x, lane = tid & 31;
    const float* s = cand_scores + (int64_t)q * k_in;
    const int32_t* ix = cand_idx + (int64_t)q * k_in;
    int32_t* out = idx_out + (int64_t)q * k;
    // the candidates come from the selections before this kernel; the output may still be
    // read by the kernel before it
    pdl_wait();
    pdl_trigger();
    // my candidates: a contiguous run of PER, in order; key 0 marks a pad (every score's
    // key is > 0 except that of a -NaN, flagged below)
    // (keys and entries stay in registers: only their thread reads them)
    const int c0 = tid * PER;
    uint32_t valid = 0u;   // bit j: candidate c0 + j is an entry
    uint32_t kor = 0u, kand = 0xFFFFFFFFu, nval = 0u;
    int32_t ent[PER];     // the candidates' entry indices
    uint32_t keys[PER];
    int r = c0 / k_in, jr = c0 - r * k_in;
#pragma unroll
    for (int j = 0; j < PER; j++) {
        const int c = c0 + j;
        uint32_t key = 0u;
        ent[j] = -1;
        if (c < n_cand) {
            const int64_t at = (int64_t)r * slice_stride + jr;
            ent[j] = ix[at];
            if (ent[j] >= 0) {
                const float v = s[at];
                if (v != v) flag(dev_status, CSA_DEV_NAN);
                key = order_key(v);
                valid |= 1u << j;
                kor |= key;
                kand &= key;
                nval++;
            }
            if (++jr == k_in) {
                jr = 0;
                r++;
            }
        }
        keys[j] = key;
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
        for (int j = 0; j < PER; j++)
            if ((valid >> j) & 1u) out[pos++] = ent[j];
        for (int j = (int)total + tid; j < k; j += kThreads) out[j] = -1;
        return;
    }
    // T, the k-th largest key, and krem, how many keys equal to T are taken
    const uint32_t vary = sh.or_and[0] ^ sh.or_and[1];
    uint32_t prefix = sh.or_and[1] & ~vary, mask = ~vary, krem = (uint32_t)k;
    int top = vary ? 31 - __clz(vary) : -1;
    bool first = true;
    while (top >= 0) {
        const int width = top >= 10 ? 11 : top + 1;
        const int shift = top + 1 - width;
        const uint32_t bmask = (1u << width) - 1u;
        for (int x = tid; x < kBins; x += kThreads) sh.hist[x] = 0u;
        __syncthreads();
        if (first) {
            // the top digits of close scores coincide: one atomic per distinct bin of a warp
#pragma unroll
            for (int j = 0; j < PER; j++) {
                const uint32_t key = keys[j];
                const uint32_t bin = (((valid >> j) & 1u) && (key & mask) == prefix)
                                         ? (key >> shift) & bmask : 0xFFFFFFFFu;
                const uint32_t peers = __match_any_sync(0xffffffffu, bin);
                if (bin != 0xFFFFFFFFu && lane == __ffs(peers) - 1)
                    atomicAdd(&sh.hist[bin], (uint32_t)__popc(peers));
            }
        } else {
#pragma unroll
            for (int j = 0; j < PER; j++) {
                const uint32_t key = keys[j];
                if (((valid >> j) & 1u) && (key & mask) == prefix)
                    atomicAdd(&sh.hist[(key >> shift) & bmask], 1u);
            }
        }
        first = false;
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
    for (int j = 0; j < PER; j++)
        if (((valid >> j) & 1u) && keys[j] == T) nt++;
    uint32_t t3;
    uint32_t ties = cta_exclusive_scan(nt, sh.scan, t3);
    uint32_t take = 0u;
#pragma unroll
    for (int j = 0; j < PER; j++) {
        if (!((valid >> j) & 1u)) continue;
        const uint32_t key = keys[j];
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
    for (int j = 0; j < PER; j++)
        if ((take >> j) & 1u) {
            if (pos < (uint32_t)k) out[pos] = ent[j];
            pos++;
        }
    if (tid == 0 && t4 != (uint32_t)k) flag(dev_status, CSA_DEV_NAN);   // no total order
}

__global__ void __launch_bounds__(256) cp_candidates_kernel(
    const int32_t* __restrict__ idx, const float* __restrict__ scores, int64_t ld,
    const int32_t* __restrict__ q_seq, const int64_t* __restrict__ lo, int B, int k,
    int32_t* __restrict__ cand_idx, float* __restrict__ cand_scores, int32_t* __restrict__ st) {
    const int q = blockIdx.x;
    // idx and the score rows come from the selection before this kernel
    pdl_wait();
    pdl_trigger();
    const int b = q_seq[q];
    const bool ok_b = b >= 0 && b < B;
    if (!ok_b && threadIdx.x == 0) flag(st, CSA_DEV_OOB);
    const int64_t base = ok_b ? lo[b] : 0;
    for (int j = threadIdx.x; j < k; j += blockDim.x) {
        const int64_t at = (int64_t)q * k + j;
        const int32_t i = idx[at];
        int32_t ci = -1;
        float cs = 0.f;
        if (i >= 0 && ok_b) {
            const int64_t gi = base + i;
            if (i < ld && base >= 0 && gi <= INT32_MAX) {
                ci = (int32_t)gi;
                cs = scores[(int64_t)q * ld + i];
            } else {
                flag(st, CSA_DEV_OOB);
            }
        }
        cand_idx[at] = ci;
        cand_scores[at] = cs;
    }
}

// One warp per output row (position j of query q).
__global__ void __launch_bounds__(256) cp_pack_rows_kernel(
    const int32_t* __restrict__ idx, const int32_t* __restrict__ q_seq,
    const int64_t* __restrict__ lo, const int64_t* __restrict__ n,
    const int64_t* __restrict__ ent_off, const uint8_t* __restrict__ entries, int64_t ent_rows,
    int row_bytes, int B, int k, int64_t rows_total, uint8_t* __restrict__ out,
    int32_t* __restrict__ local_idx, int32_t* __restrict__ st) {
    const int lane = threadIdx.x & 31;
    const int64_t r = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
    // idx comes from the merge before this kernel; `out` may still be read by the kernel
    // before it
    pdl_wait();
    pdl_trigger();
    if (r >= rows_total) return;
    const int q = (int)(r / k);
    const int32_t i = idx[r];
    const int b = q_seq[q];
    const int4* src = nullptr;
    if (i >= 0) {
        if (b >= 0 && b < B) {
            const int64_t local = (int64_t)i - lo[b];
            if (local >= 0 && local < n[b]) {
                const int64_t row = ent_off[b] + local;
                if (row >= 0 && row < ent_rows)
                    src = reinterpret_cast<const int4*>(entries + row * row_bytes);
                else if (lane == 0)
                    flag(st, CSA_DEV_OOB);
            }
        } else if (lane == 0) {
            flag(st, CSA_DEV_OOB);
        }
    }
    if (local_idx && lane == 0) local_idx[r] = i >= 0 ? (int32_t)(r - (int64_t)q * k) : -1;
    int4* dst = reinterpret_cast<int4*>(out + r * row_bytes);
    const int n16 = row_bytes >> 4;
    for (int c = lane; c < n16; c += 32) dst[c] = src ? __ldg(src + c) : make_int4(0, 0, 0, 0);
}

}  // namespace

bool topk_merge_supported(int n_cand, int k) { return n_cand >= 1 && n_cand <= kMaxCand && k >= 1; }

cudaError_t launch_topk_merge(const float* cand_scores, const int32_t* cand_idx,
                              int64_t slice_stride, int W, int Q, int k_in, int k,
                              int32_t* idx_out, int32_t* st, cudaStream_t stream) {
    if (Q == 0) return cudaSuccess;
    const int n_cand = W * k_in;
    const size_t smem = sizeof(MergeShared);
    auto kernel = n_cand <= kThreads * 4   ? topk_merge_kernel<4>
                  : n_cand <= kThreads * 8 ? topk_merge_kernel<8>
                                           : topk_merge_kernel<16>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    LaunchScope scope(kKTopkMerge, stream);
    return launch_pdl(kernel, dim3(Q), dim3(kThreads), smem, stream, cand_scores, cand_idx,
                      slice_stride, k_in, n_cand, k, idx_out, st);
}

cudaError_t launch_cp_candidates(const int32_t* idx, const float* scores, int64_t ld,
                                 const int32_t* q_seq, const int64_t* lo, int Q, int B, int k,
                                 int32_t* cand_idx, float* cand_scores, int32_t* st,
                                 cudaStream_t stream) {
    if (Q == 0) return cudaSuccess;
    LaunchScope scope(kKCpCandidates, stream);
    return launch_pdl(cp_candidates_kernel, dim3(Q), dim3(256), 0, stream, idx, scores, ld,
                      q_seq, lo, B, k, cand_idx, cand_scores, st);
}

cudaError_t launch_cp_pack_rows(const int32_t* idx, const int32_t* q_seq, const int64_t* lo,
                                const int64_t* n, const int64_t* ent_off,
                                const uint8_t* entries, int64_t ent_rows, int row_bytes, int Q,
                                int B, int k, uint8_t* out, int32_t* local_idx, int32_t* st,
                                cudaStream_t stream) {
    const int64_t rows = (int64_t)Q * k;
    if (rows == 0) return cudaSuccess;
    LaunchScope scope(kKCpPackRows, stream);
    const int64_t blocks = (rows + 7) / 8;
    return launch_pdl(cp_pack_rows_kernel, dim3((unsigned)blocks), dim3(256), 0, stream, idx,
                      q_seq, lo, n, ent_off, entries, ent_rows, row_bytes, B, k, rows, out, local_idx,
                      st);
}

}  // namespace csa
