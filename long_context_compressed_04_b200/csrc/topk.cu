// Step a4: per-query top-k over the indexer scores.
//
// "DeepSeek-V4 深度分析报告" 2.1 CSA: keep the k best compressed entries per query
// (k = 512 / 1024).  The selection order is total: larger score first, lower entry index
// first among equal scores (-0 and +0 are equal), so the selected set is unique and does
// not depend on how the work is partitioned -- the result is batch-invariant by
// construction.
//
// One CTA (1024 threads) per query, scores mapped to order-preserving 32-bit keys.  The
// goal is the k-th largest key T and the number of keys equal to T to take.
//  0. Rows of up to 44K scores are staged in shared memory as keys (bulk copies); the OR
//     and AND of all keys give the bits every key shares.  Rows much longer than k first
//     try a bound B from a fixed strided sample of 1024 keys (the lower edge of the digit
//     bin holding the sample's ~(2k * 1024 / n)-th largest): one marking pass finds the
//     keys >= B; if they number between k and 4096 they hold the k largest, T is selected
//     among them alone and the output is written from the marks (as in 4).  Otherwise:
//  1. The radix starts at the highest bit that varies (scores of one query share sign and
//     most exponent bits, and a fixed first digit would put nearly all of them in one bin).
//  2. An 11-bit histogram of that digit (shared-memory atomics) and a block-wide scan over
//     the bins, from the top, give the bin holding the k-th key.
//  3. Keys in that bin are compacted to a short candidate list (if it fits; one shared
//     atomic per warp and key slot), and the remaining bits are resolved on the list;
//     otherwise further full passes run.
//  4. A marking pass stores, per 32 consecutive entries, the ballot words of keys > T and
//     keys == T.  One block-wide scan over the words gives each its output offset and tie
//     rank; every key > T and the first needed keys == T are written from the words' bits
//     in ascending entry order, so the indices come out already sorted.
//
// Rows too long for one CTA's shared memory (1M-token contexts: 262144 entries) run one
// thread-block cluster of up to 8 CTAs per query instead; rank r owns a contiguous slice of
// the row.  Each digit's histogram is summed across the cluster through distributed shared
// memory, so every rank picks the same bin.  As soon as the chosen bin holds at most 4096
// keys of the row, one exchange gives every rank all ranks' candidates and their counts of
// keys above the bin; the remaining bits are then resolved on every rank alone, and the
// lower ranks' counts give each rank its output offset and tie budget.
#include <algorithm>

#include "launchers.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kThreads = 1024;
constexpr int kWarps = kThreads / 32;
constexpr int kBins = 2048;
constexpr int kChunk = 4 * kThreads;
constexpr int kMaxCand = 4096;

__device__ __forceinline__ uint32_t score_key(float s) { return order_key(s); }

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

struct Shared {
    uint32_t hist[kBins];
    uint32_t scan_tmp[33];
    unsigned long long scan64[33];
    uint32_t bin, krem, key_or, key_and, ncand;
    uint32_t s_or, s_and, c_or, c_and;   // OR / AND of the sample and of the candidates
    uint64_t stage_bar;                   // bulk copies of the row into shared memory
    int abort;
    uint32_t cor[2], ngrp, nsel;          // the group path (see topk_by_groups)
    uint32_t cand[kMaxCand];
};


// Exclusive prefix sum over the CTA of a 64-bit `v`; `total` gets the CTA sum.
__device__ __forceinline__ unsigned long long block_exclusive_scan64(unsigned long long v,
                                                                     unsigned long long* tmp,
                                                                     unsigned long long& total) {
    const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
    unsigned long long x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const unsigned long long y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) tmp[wid] = x;
    __syncthreads();
    if (wid == 0) {
        const unsigned long long wv = lane < kWarps ? tmp[lane] : 0ull;
        unsigned long long inc = wv;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const unsigned long long y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        __syncwarp();
        tmp[lane] = inc - wv;
        if (lane == 31) tmp[32] = inc;
    }
    __syncthreads();
    const unsigned long long res = x - v + tmp[wid];
    total = tmp[32];
    __syncthreads();
    return res;
}

__device__ __forceinline__ uint32_t lanemask_lt() {
    uint32_t m;
    asm("mov.u32 %0, %%lanemask_lt;" : "=r"(m));
    return m;
}

// Over the counts `h` of the current digit: picks the bin holding the krem-th largest key
// (bins scanned from the top) and the rank left inside it; 1024 threads, 2 bins each.
__device__ __forceinline__ void pick_bin_in(const uint32_t* h, uint32_t* scan_tmp,
                                            uint32_t* bin_out, uint32_t* krem_out,
                                            uint32_t& krem) {
    const int tid = threadIdx.x;
    const int bhi = kBins - 1 - 2 * tid, blo = bhi - 1;
    const uint32_t chi = h[bhi], clo = h[blo];
    uint32_t tot;
    const uint32_t above = block_exclusive_scan(chi + clo, scan_tmp, tot);
    if (above < krem && krem <= above + chi) {
        *bin_out = (uint32_t)bhi;
        *krem_out = krem - above;
    } else if (above + chi < krem && krem <= above + chi + clo) {
        *bin_out = (uint32_t)blo;
        *krem_out = krem - above - chi;
    }
    __syncthreads();
    krem = *krem_out;
}

// After hist[] holds the counts of the current digit: picks the bin holding the krem-th
// largest key (bins scanned from the top) and the rank left inside it.
__device__ __forceinline__ void pick_bin(Shared& sh, uint32_t& krem) {
    const int tid = threadIdx.x;
    const int bhi = kBins - 1 - 2 * tid, blo = bhi - 1;
    const uint32_t chi = sh.hist[bhi], clo = sh.hist[blo];
    uint32_t tot;
    const uint32_t above = block_exclusive_scan(chi + clo, sh.scan_tmp, tot);
    if (above < krem && krem <= above + chi) {
        sh.bin = (uint32_t)bhi;
        sh.krem = krem - above;
    } else if (above + chi < krem && krem <= above + chi + clo) {
        sh.bin = (uint32_t)blo;
        sh.krem = krem - above - chi;
    }
    __syncthreads();
    krem = sh.krem;
}

// The kth largest (1-based, kth <= cnt) of the cnt keys list[0 .. cnt) in shared memory,
// whose OR and AND are kor / kand: 11-bit radix digits from the highest bit that varies;
// `krem` gets the number of keys equal to it that the kth largest include.  All threads
// call it; it ends with the CTA synchronised.
__device__ __forceinline__ uint32_t select_kth_list(Shared& sh, const uint32_t* list,
                                                    uint32_t cnt, uint32_t kth, uint32_t kor,
                                                    uint32_t kand, uint32_t& krem) {
    const uint32_t vary = kor ^ kand;
    uint32_t prefix = kand & ~vary, mask = ~vary;
    krem = kth;
    int top = vary ? 31 - __clz(vary) : -1;
    while (top >= 0) {
        const int width = top >= 10 ? 11 : top + 1;
        const int shift = top + 1 - width;
        const uint32_t bmask = (1u << width) - 1u;
        for (int x = threadIdx.x; x < kBins; x += kThreads) sh.hist[x] = 0u;
        __syncthreads();
        for (uint32_t c = threadIdx.x; c < cnt; c += kThreads) {
            const uint32_t key = list[c];
            if ((key & mask) == prefix) atomicAdd(&sh.hist[(key >> shift) & bmask], 1u);
        }
        __syncthreads();
        pick_bin(sh, krem);
        prefix |= sh.bin << shift;
        mask |= bmask << shift;
        top = shift - 1;
        __syncthreads();
    }
    return prefix;
}

// As select_kth_list, over shared-memory scratch given by pointers: hist >= kBins words,
// scan_tmp >= 33 words, bin_out / krem_out one word each.  With max_digits > 0 it stops
// after that many digits and returns the lower edge of the bin reached, a value <= the kth
// largest (krem is then not meaningful).
__device__ __forceinline__ uint32_t select_kth_raw(const uint32_t* list, uint32_t cnt, uint32_t kth,
                                                   uint32_t kor, uint32_t kand, uint32_t& krem,
                                                   uint32_t* hist, uint32_t* scan_tmp,
                                                   uint32_t* bin_out, uint32_t* krem_out,
                                                   int max_digits = 0) {
    const uint32_t vary = kor ^ kand;
    uint32_t prefix = kand & ~vary, mask = ~vary;
    krem = kth;
    int top = vary ? 31 - __clz(vary) : -1;
    for (int digit = 0; top >= 0 && (max_digits == 0 || digit < max_digits); digit++) {
        const int width = top >= 10 ? 11 : top + 1;
        const int shift = top + 1 - width;
        const uint32_t bmask = (1u << width) - 1u;
        for (int x = threadIdx.x; x < kBins; x += kThreads) hist[x] = 0u;
        __syncthreads();
        for (uint32_t c = threadIdx.x; c < cnt; c += kThreads) {
            const uint32_t key = list[c];
            if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & bmask], 1u);
        }
        __syncthreads();
        pick_bin_in(hist, scan_tmp, bin_out, krem_out, krem);
        prefix |= *bin_out << shift;
        mask |= bmask << shift;
        top = shift - 1;
        __syncthreads();
    }
    return prefix;
}

// Shared memory of the group path (see topk_by_groups): two words per group of 32 entries
// (the group keys and the list of groups reaching the bound, later the selection words),
// then cap candidate keys and cap candidate entries.
__host__ __device__ constexpr size_t group_smem_bytes(int max_n, int cap) {
    // group keys and list, candidates (key, entry), then the output words (2 x 2k = cap)
    return (size_t)((2 * ((max_n + 31) / 32) + 3) / 4) * 16 + (size_t)cap * 12;
}

// OR / AND of `v` over the CTA into or_and[0] / or_and[1] (initialised by the caller before
// a barrier); ends with the CTA synchronised.
__device__ __forceinline__ void block_or_and(uint32_t o, uint32_t a, uint32_t* or_and) {
#pragma unroll
    for (int s = 16; s > 0; s >>= 1) {
        o |= __shfl_xor_sync(0xffffffffu, o, s);
        a &= __shfl_xor_sync(0xffffffffu, a, s);
    }
    if ((threadIdx.x & 31) == 0) {
        atomicOr(&or_and[0], o);
        atomicAnd(&or_and[1], a);
    }
    __syncthreads();
}

// Top-k of a query from the group maxima the indexer wrote: qg[g] is the largest score key
// of entries 32g .. 32g + 31.  B, the k-th largest of the G = ceil(n / 32) group keys (one
// needs G >= k), bounds the k-th largest score from below, since the k groups at or above B
// each hold an entry whose key is >= B.  So the top-k are among the entries >= B, and those
// lie in the groups whose key is >= B (about k of them): only those groups' scores are
// read.  The entries >= B are listed (at least k of them; the call returns false, with
// nothing written, when more than cap, or when more than 2k groups reach B), the k-th
// largest key T is selected among them, and the selection -- every entry > T and the
// lowest-indexed ties -- is written in ascending entry order from bit words over the
// listed groups.  The result is the unique top-k under the tie order.  All 1024 threads
// call it (for G >= 2k); dyn holds group_smem_bytes(n, cap) bytes.
__device__ bool topk_by_groups(const float* __restrict__ s, bool vec,
                               const uint32_t* __restrict__ qg, int n, int k, int cap,
                               int32_t* __restrict__ out, uint8_t* dyn, Shared& sh) {
    const int tid = threadIdx.x, lane = tid & 31;
    const int G = (n + 31) >> 5;
    uint32_t* gk = reinterpret_cast<uint32_t*>(dyn);
    uint32_t* glist = gk + G;
    uint32_t* ckey = reinterpret_cast<uint32_t*>(dyn + ((2 * G + 3) / 4) * 16);
    uint32_t* cent = ckey + cap;
    // 1. the group keys
    if (tid == 0) {
        sh.cor[0] = 0u;
        sh.cor[1] = 0xFFFFFFFFu;
        sh.ngrp = 0u;
        sh.nsel = 0u;
    }
    __syncthreads();
    uint32_t kor = 0u, kand = 0xFFFFFFFFu;
    {
        // 16-byte loads when the row is aligned (all of a thread's loads in flight)
        const int G4 = (reinterpret_cast<uintptr_t>(qg) & 15) == 0 ? G >> 2 : 0;
#pragma unroll 4
        for (int g4 = tid; g4 < G4; g4 += kThreads) {
            const uint4 v = reinterpret_cast<const uint4*>(qg)[g4];
            reinterpret_cast<uint4*>(gk)[g4] = v;
            kor |= v.x | v.y | v.z | v.w;
            kand &= v.x & v.y & v.z & v.w;
        }
        for (int g = 4 * G4 + tid; g < G; g += kThreads) {
            const uint32_t v = qg[g];
            gk[g] = v;
            kor |= v;
            kand &= v;
        }
    }
    block_or_and(kor, kand, sh.cor);
    // 2. B: the lower edge of the bin of the k-th largest group key after two 11-bit
    // digits from the highest varying bit (a lower bound of it, as exact as needed)
    uint32_t krem;
    const uint32_t B = select_kth_raw(gk, (uint32_t)G, (uint32_t)k, sh.cor[0], sh.cor[1], krem,
                                      sh.hist, sh.scan_tmp, &sh.bin, &sh.krem, 2);
    // 3. the groups reaching B, in ascending order: each thread a contiguous run of groups,
    // placed by one block scan (the output below walks them in this order)
    {
        // runs of a multiple of 4 groups, read as 16-byte vectors (gk is 16-byte aligned)
        const int per = ((G + kThreads - 1) / kThreads + 3) & ~3;
        const int g0 = tid * per, g1 = min(G, g0 + per);
        uint32_t cnt = 0u;
        for (int g = g0; g < g1; g += 4) {
            const uint4 v = *reinterpret_cast<const uint4*>(gk + g);
            cnt += (v.x >= B) + (g + 1 < g1 && v.y >= B) + (g + 2 < g1 && v.z >= B) +
                   (g + 3 < g1 && v.w >= B);
        }
        unsigned long long tot;
        uint32_t pos = (uint32_t)block_exclusive_scan64(cnt, sh.scan64, tot);
        // the list, and in gk (no longer needed) each listed group's position in it
        for (int g = g0; g < g1; g += 4) {
            const uint4 v = *reinterpret_cast<const uint4*>(gk + g);
            const uint32_t vv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
            for (int z = 0; z < 4; z++)
                if (g + z < g1 && vv[z] >= B) {
                    glist[pos] = (uint32_t)(g + z);
                    gk[g + z] = pos++;
                }
        }
        if (tid == 0) sh.ngrp = (uint32_t)tot;
        __syncthreads();
    }
    const uint32_t ng = sh.ngrp;
    // the output words below cover the listed groups only: more than 2k of them (massive
    // ties among the group keys) take the full row instead
    if (ng > 2u * (uint32_t)k) return false;
    if (tid == 0) sh.nsel = 0u;
    __syncthreads();
    // 4. their entries reaching B: 8 slots of 4 entries per group, up to kGatherSlots slots
    // per thread with all of their loads in flight; each thread's passing entries are
    // placed by one warp scan and one shared atomic per warp
    constexpr int kGatherSlots = 4;
    const uint32_t nslots = ng * 8u;
    for (uint32_t b0 = 0; b0 < nslots; b0 += (uint32_t)(kGatherSlots * kThreads)) {
        uint32_t key[kGatherSlots][4] = {};
        int e0[kGatherSlots];
#pragma unroll
        for (int u = 0; u < kGatherSlots; u++) {
            const uint32_t slot = b0 + (uint32_t)tid + (uint32_t)(u * kThreads);
            e0[u] = slot < nslots ? (int)(glist[slot >> 3] * 32u + (slot & 7u) * 4u) : n;
            if (e0[u] < n) load4(s, e0[u], n, vec, key[u]);
        }
        uint32_t pm = 0u;   // bit 4u + z: entry e0[u] + z reaches B
#pragma unroll
        for (int u = 0; u < kGatherSlots; u++)
#pragma unroll
            for (int z = 0; z < 4; z++)
                if (e0[u] + z < n && key[u][z] >= B) pm |= 1u << (4 * u + z);
        const uint32_t cnt = __popc(pm);
        uint32_t inc = cnt;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
            if (lane >= o) inc += y;
        }
        uint32_t base = 0u;
        if (lane == 31 && inc) base = atomicAdd(&sh.nsel, inc);
        base = __shfl_sync(0xffffffffu, base, 31);
        uint32_t pos = base + inc - cnt;
#pragma unroll
        for (int u = 0; u < kGatherSlots; u++)
#pragma unroll
            for (int z = 0; z < 4; z++)
                if ((pm >> (4 * u + z)) & 1u) {
                    if (pos < (uint32_t)cap) {
                        ckey[pos] = key[u][z];
                        cent[pos] = (uint32_t)(e0[u] + z);
                    }
                    pos++;
                }
    }
    if (tid == 0) {
        sh.cor[0] = 0u;
        sh.cor[1] = 0xFFFFFFFFu;
    }
    __syncthreads();
    const uint32_t c = sh.nsel;
    // the same value in every thread; fewer than k only if some group maximum was not
    // written (an entry row past the key store, flagged by the indexer)
    if (c > (uint32_t)cap || c < (uint32_t)k) return false;
    // 5. T among the c >= k candidates
    kor = 0u;
    kand = 0xFFFFFFFFu;
    for (uint32_t i = tid; i < c; i += kThreads) {
        kor |= ckey[i];
        kand &= ckey[i];
    }
    block_or_and(kor, kand, sh.cor);
    const uint32_t T = select_kth_raw(ckey, c, (uint32_t)k, sh.cor[0], sh.cor[1], krem,
                                      sh.hist, sh.scan_tmp, &sh.bin, &sh.krem);
    // 6. selection words over the listed groups (ascending): bit e & 31 of word gk[e >> 5]
    // for every candidate > T (selw) or == T (tiew); each thread a contiguous run of words,
    // placed by one block scan of (selected, tied) counts, every entry > T and the first
    // krem ties written in ascending entry order
    uint32_t* selw = cent + cap;
    uint32_t* tiew = selw + 2 * k;
    for (uint32_t w = tid; w < ng; w += kThreads) {
        selw[w] = 0u;
        tiew[w] = 0u;
    }
    __syncthreads();
    for (uint32_t i = tid; i < c; i += kThreads) {
        const uint32_t key = ckey[i], e = cent[i];
        if (key > T) atomicOr(&selw[gk[e >> 5]], 1u << (e & 31));
        else if (key == T) atomicOr(&tiew[gk[e >> 5]], 1u << (e & 31));
    }
    __syncthreads();
    {
        const uint32_t per = (ng + kThreads - 1) / kThreads;
        const uint32_t w0 = (uint32_t)tid * per, w1 = min(ng, w0 + per);
        uint32_t cs = 0u, ct = 0u;
        for (uint32_t w = w0; w < w1; w++) {
            cs += __popc(selw[w]);
            ct += __popc(tiew[w]);
        }
        unsigned long long tot;
        const unsigned long long pre =
            block_exclusive_scan64(((unsigned long long)cs << 32) | ct, sh.scan64, tot);
        uint32_t ties = (uint32_t)pre;
        uint32_t pos = (uint32_t)(pre >> 32) + min(ties, krem);
        for (uint32_t w = w0; w < w1; w++) {
            const uint32_t sw = selw[w], tw = tiew[w];
            uint32_t take_t = 0u;
            if (ties < krem) {
                uint32_t need = krem - ties, tt = tw;
                while (need && tt) {
                    take_t |= tt & (0u - tt);
                    tt &= tt - 1u;
                    need--;
                }
            }
            ties += __popc(tw);
            uint32_t take = sw | take_t;
            const int32_t base = (int32_t)(glist[w] << 5);
            while (take) {
                const int bit = __ffs(take) - 1;
                if (pos < (uint32_t)k) out[pos] = base + bit;
                pos++;
                take &= take - 1;
            }
        }
    }
    return true;
}

// STAGED: the query's row is first copied to shared memory as keys (16-byte loads, eight in
// flight per thread) and every pass reads it from there.
template <bool STAGED>
__global__ void __launch_bounds__(kThreads) topk_radix_kernel(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ q_seq,
    const int32_t* __restrict__ q_pos, const int64_t* __restrict__ seq_len, int B, int m,
    int max_n, int k, int32_t* __restrict__ idx_out, int32_t* __restrict__ dev_status,
    const uint32_t* __restrict__ gmax, int64_t ld_g, int cap) {
    using namespace sm100;
    __shared__ Shared sh;
    const int qq = blockIdx.x;
    const int tid = threadIdx.x, lane = tid & 31;
    const int b = q_seq[qq];
    const int t = q_pos[qq];
    // invalid queries (flagged by the scoring kernel) select nothing
    const bool valid = b >= 0 && b < B && t >= 0 && (int64_t)t < seq_len[b];
    pdl_wait();   // scores come from the indexer
    pdl_trigger();
    int n = valid ? (t + 1) / m : 0;
    if (n > max_n) n = max_n;  // capacity already flagged by the scoring kernel
    const float* s = scores + (int64_t)qq * ld;
    int32_t* out = idx_out + (int64_t)qq * k;
    if (n <= k) {
        for (int j = tid; j < k; j += kThreads) out[j] = j < n ? j : -1;
        return;
    }
    bool vec = (reinterpret_cast<uintptr_t>(s) & 15) == 0;
    if (gmax && ((n + 31) >> 5) >= 2 * k) {
        // from the indexer's group maxima (see topk_by_groups); the full row below only if
        // more than cap entries reach the bound.  With fewer than 2k groups the bound is
        // the maximum of nearly every group and admits most of the row, so the row's own
        // selection is taken straight away.
        extern __shared__ uint4 dyn_g[];
        if (topk_by_groups(s, vec, gmax + (int64_t)qq * ld_g, n, k, cap, out,
                           reinterpret_cast<uint8_t*>(dyn_g), sh))
            return;
    }
    if (tid == 0) {
        sh.key_or = 0u;
        sh.key_and = 0xFFFFFFFFu;
        sh.ncand = 0u;
        sh.s_or = sh.c_or = 0u;
        sh.s_and = sh.c_and = 0xFFFFFFFFu;
    }
    __syncthreads();
    uint32_t kor = 0u, kand = 0xFFFFFFFFu;
    // dynamic shared memory: the selection words (2 per 32 entries), then the staged keys
    extern __shared__ uint4 dyn4[];
    const int nwords = (n + 31) >> 5;
    uint32_t* selw = reinterpret_cast<uint32_t*>(dyn4);
    uint32_t* tiew = selw + ((max_n + 31) >> 5);
    uint4* skey4 = dyn4 + ((2 * ((max_n + 31) >> 5) + 3) >> 2);
    const uint32_t* skey = reinterpret_cast<const uint32_t*>(skey4);
    // keys of entries i .. i+3 (0 past n) and of entry i
    auto get4 = [&](int i, uint32_t* key) {
        if constexpr (STAGED) {
            // only the staged part of the row is read (past n the buffer may end)
            const uint4 v = i < n ? skey4[i >> 2] : make_uint4(0u, 0u, 0u, 0u);
            key[0] = i < n ? v.x : 0u;
            key[1] = i + 1 < n ? v.y : 0u;
            key[2] = i + 2 < n ? v.z : 0u;
            key[3] = i + 3 < n ? v.w : 0u;
        } else {
            load4(s, i, n, vec, key);
        }
    };
    auto get1 = [&](int i) -> uint32_t {
        if constexpr (STAGED) {
            return skey[i];
        } else {
            return score_key(s[i]);
        }
    };
    if constexpr (STAGED) {
      if (vec) {
        // the whole row in flight at once: bulk copies (8 KB each, one per lane of warp 0)
        // straight into shared memory, then one pass turns the scores into keys in place
        const int n4 = n >> 2;
        const uint32_t bytes = (uint32_t)n4 * 16u;
        if (tid == 0) {
            mbar_init(&sh.stage_bar, 1);
            mbar_fence_init();
            sh.abort = 0;
        }
        __syncthreads();
        if (tid < 32) {
            if (lane == 0) mbar_arrive_expect_tx(&sh.stage_bar, bytes);
            __syncwarp();
            constexpr uint32_t kPiece = 8192;
            for (uint32_t off = (uint32_t)lane * kPiece; off < bytes; off += 32 * kPiece)
                bulk_load(reinterpret_cast<uint8_t*>(skey4) + off,
                          reinterpret_cast<const uint8_t*>(s) + off, min(kPiece, bytes - off),
                          &sh.stage_bar);
        }
        if (!named_barrier_and(1, kThreads, mbar_wait(&sh.stage_bar, 0, &sh.abort, dev_status))) {
            // timed out (flagged): let the copies drain before the CTA leaves
            mbar_drain(&sh.stage_bar, 0, dev_status);
            return;
        }
        for (int j = tid; j < ((n + 3) >> 2); j += kThreads) {
            float e[4];
            if (j < n4) {
                const uint4 v = skey4[j];
                e[0] = __uint_as_float(v.x);
                e[1] = __uint_as_float(v.y);
                e[2] = __uint_as_float(v.z);
                e[3] = __uint_as_float(v.w);
            } else {
#pragma unroll
                for (int z = 0; z < 4; z++) e[z] = 4 * j + z < n ? s[4 * j + z] : 0.f;
            }
            uint32_t kk[4];
#pragma unroll
            for (int z = 0; z < 4; z++) {
                kk[z] = score_key(e[z]);
                if (4 * j + z < n) {
                    kor |= kk[z];
                    kand &= kk[z];
                }
            }
            skey4[j] = make_uint4(kk[0], kk[1], kk[2], kk[3]);
        }
      } else {
        constexpr int kBatch = 8;
        for (int i0 = 4 * tid; i0 < n; i0 += 4 * kThreads * kBatch) {
            float4 v[kBatch];
#pragma unroll
            for (int u = 0; u < kBatch; u++) {
                const int i = i0 + u * 4 * kThreads;
                if (vec && i + 3 < n) {
                    v[u] = *reinterpret_cast<const float4*>(s + i);
                } else {
                    v[u].x = i < n ? s[i] : 0.f;
                    v[u].y = i + 1 < n ? s[i + 1] : 0.f;
                    v[u].z = i + 2 < n ? s[i + 2] : 0.f;
                    v[u].w = i + 3 < n ? s[i + 3] : 0.f;
                }
            }
#pragma unroll
            for (int u = 0; u < kBatch; u++) {
                const int i = i0 + u * 4 * kThreads;
                const float e[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
                uint32_t kk[4];
#pragma unroll
                for (int z = 0; z < 4; z++) {
                    kk[z] = score_key(e[z]);
                    if (i + z < n) {
                        kor |= kk[z];
                        kand &= kk[z];
                    }
                }
                if (i < n) skey4[i >> 2] = make_uint4(kk[0], kk[1], kk[2], kk[3]);
            }
        }
      }
    } else {
        for (int c0 = 0; c0 < n; c0 += kChunk) {
            uint32_t key[4];
            load4(s, c0 + 4 * tid, n, vec, key);
#pragma unroll
            for (int u = 0; u < 4; u++) {
                if (c0 + 4 * tid + u < n) {
                    kor |= key[u];
                    kand &= key[u];
                }
            }
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kor |= __shfl_xor_sync(0xffffffffu, kor, o);
        kand &= __shfl_xor_sync(0xffffffffu, kand, o);
    }
    if (lane == 0) {
        atomicOr(&sh.key_or, kor);
        atomicAnd(&sh.key_and, kand);
    }
    __syncthreads();
    const uint32_t diff = sh.key_or ^ sh.key_and;   // bits that vary across the row
    const int wid = tid >> 5;
    if constexpr (STAGED) {
        // Rows much longer than k: a bound B from a fixed strided sample of the row, chosen so
        // that about 2k keys of the row are >= B.  One pass marks the keys >= B in words of 32
        // entries; if they number between k and kMaxCand they hold the k largest, which are
        // then selected among them alone and written from the words.  The sample only decides
        // how fast the unique result is found: otherwise the general passes below run.
        const long long r_ll = (2LL * k * kThreads + n - 1) / n + 8;
        if (diff != 0u && r_ll <= kThreads / 2) {
            // B: the lower edge of the bin (of one 11-bit digit from the sample's highest
            // varying bit) that holds the sample's r-th largest key; at least r keys are >= B
            const uint32_t sv = skey[(int)(((long long)tid * n) / kThreads)];
            {
                uint32_t so = sv, sa = sv;
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    so |= __shfl_xor_sync(0xffffffffu, so, o);
                    sa &= __shfl_xor_sync(0xffffffffu, sa, o);
                }
                if (lane == 0) {
                    atomicOr(&sh.s_or, so);
                    atomicAnd(&sh.s_and, sa);
                }
            }
            for (int x = tid; x < kBins; x += kThreads) sh.hist[x] = 0u;
            __syncthreads();
            const uint32_t svary = sh.s_or ^ sh.s_and;
            uint32_t B = sh.s_and;   // all sample keys equal
            if (svary) {
                const int stop = 31 - __clz(svary);
                const int width = stop >= 10 ? 11 : stop + 1;
                const int shift = stop + 1 - width;
                atomicAdd(&sh.hist[(sv >> shift) & ((1u << width) - 1u)], 1u);
                __syncthreads();
                uint32_t rk = (uint32_t)r_ll;
                pick_bin(sh, rk);
                const uint32_t hi = stop >= 31 ? 0u : (sh.s_and >> (stop + 1)) << (stop + 1);
                B = hi | (sh.bin << shift);
            }
            for (int r = wid; r < nwords; r += kWarps) {
                const int i = (r << 5) + lane;
                const bool in = i < n;
                const uint32_t key = in ? skey[i] : 0u;
                const uint32_t ge = __ballot_sync(0xffffffffu, in && key >= B);
                if (lane == 0) selw[r] = ge;
            }
            __syncthreads();
            const int wpt = (nwords + kThreads - 1) / kThreads;
            const int w0 = min(tid * wpt, nwords), w1 = min(w0 + wpt, nwords);
            uint32_t cnt = 0;
            for (int w = w0; w < w1; w++) cnt += __popc(selw[w]);
            uint32_t total;
            uint32_t off = block_exclusive_scan(cnt, sh.scan_tmp, total);
            if (total >= (uint32_t)k && total <= (uint32_t)kMaxCand) {
                // the candidates' keys, in entry order, and their OR / AND
                uint32_t co = 0u, ca = 0xFFFFFFFFu;
                for (int w = w0; w < w1; w++) {
                    uint32_t bits = selw[w];
                    while (bits) {
                        const int bit = __ffs(bits) - 1;
                        const uint32_t key = skey[(w << 5) + bit];
                        sh.cand[off++] = key;
                        co |= key;
                        ca &= key;
                        bits &= bits - 1;
                    }
                }
#pragma unroll
                for (int o = 16; o > 0; o >>= 1) {
                    co |= __shfl_xor_sync(0xffffffffu, co, o);
                    ca &= __shfl_xor_sync(0xffffffffu, ca, o);
                }
                if (lane == 0) {
                    atomicOr(&sh.c_or, co);
                    atomicAnd(&sh.c_and, ca);
                }
                __syncthreads();
                uint32_t kr;
                const uint32_t T =
                    select_kth_list(sh, sh.cand, total, (uint32_t)k, sh.c_or, sh.c_and, kr);
                // keys > T and the first kr keys == T, in entry order: per thread its words'
                // counts, one 64-bit scan (ties high, keys > T low), then the writes
                uint32_t cg = 0, ce = 0;
                for (int w = w0; w < w1; w++) {
                    uint32_t bits = selw[w];
                    while (bits) {
                        const uint32_t key = skey[(w << 5) + __ffs(bits) - 1];
                        cg += key > T;
                        ce += key == T;
                        bits &= bits - 1;
                    }
                }
                unsigned long long tot;
                const unsigned long long pre =
                    block_exclusive_scan64(((unsigned long long)ce << 32) | cg, sh.scan64, tot);
                uint32_t ties = (uint32_t)(pre >> 32);
                uint32_t pos = (uint32_t)pre + min(ties, kr);
                for (int w = w0; w < w1; w++) {
                    uint32_t bits = selw[w];
                    while (bits) {
                        const int bit = __ffs(bits) - 1;
                        const uint32_t key = skey[(w << 5) + bit];
                        bool take = key > T;
                        if (key == T) take = ties++ < kr;
                        if (take) {
                            if (pos < (uint32_t)k) out[pos] = (w << 5) + bit;
                            pos++;
                        }
                        bits &= bits - 1;
                    }
                }
                // the row's total; NaN scores (no total order) break it
                if (tid == 0 && (uint32_t)tot + min((uint32_t)(tot >> 32), kr) != (uint32_t)k)
                    flag(dev_status, CSA_DEV_NAN);
                return;
            }
            __syncthreads();   // the general passes reuse the shared state
        }
    }
    uint32_t prefix = sh.key_and & ~diff;           // = the bits all keys share
    uint32_t mask = ~diff;
    uint32_t krem = (uint32_t)k;
    // digits from the highest varying bit down, 11 bits at a time
    int top = diff ? 31 - __clz(diff) : -1;
    bool compacted = false;
    while (top >= 0) {
        const int width = top >= 10 ? 11 : top + 1;
        const int shift = top + 1 - width;
        const uint32_t bmask = (1u << width) - 1u;
        for (int x = tid; x < kBins; x += kThreads) sh.hist[x] = 0u;
        __syncthreads();
        if (!compacted) {
            for (int c0 = 0; c0 < n; c0 += kChunk) {
                uint32_t key[4];
                get4(c0 + 4 * tid, key);
#pragma unroll
                for (int u = 0; u < 4; u++)
                    if (c0 + 4 * tid + u < n && (key[u] & mask) == prefix)
                        atomicAdd(&sh.hist[(key[u] >> shift) & bmask], 1u);
            }
        } else {
            for (uint32_t c = tid; c < sh.ncand; c += kThreads) {
                const uint32_t key = sh.cand[c];
                if ((key & mask) == prefix) atomicAdd(&sh.hist[(key >> shift) & bmask], 1u);
            }
        }
        __syncthreads();
        pick_bin(sh, krem);
        const uint32_t bin = sh.bin;
        const uint32_t in_bin = sh.hist[bin];
        prefix |= bin << shift;
        mask |= bmask << shift;
        top = shift - 1;
        __syncthreads();
        if (!compacted && top >= 0 && in_bin <= (uint32_t)kMaxCand) {
            // keys in the chosen bin become the candidate list for the remaining bits (one
            // shared atomic per warp and key slot)
            for (int c0 = 0; c0 < n; c0 += kChunk) {
                uint32_t key[4];
                get4(c0 + 4 * tid, key);
#pragma unroll
                for (int u = 0; u < 4; u++) {
                    const bool p = c0 + 4 * tid + u < n && (key[u] & mask) == prefix;
                    const uint32_t bal = __ballot_sync(0xffffffffu, p);
                    uint32_t slot = 0;
                    if (lane == 0 && bal) slot = atomicAdd(&sh.ncand, (uint32_t)__popc(bal));
                    slot = __shfl_sync(0xffffffffu, slot, 0);
                    if (p) sh.cand[slot + __popc(bal & lanemask_lt())] = key[u];
                }
            }
            compacted = true;
            __syncthreads();
        }
    }
    const uint32_t T = prefix;   // the k-th largest key; krem keys equal to T are taken
    // marking: word r holds the entries 32 r .. 32 r + 31 (bit = lane)
    for (int r = wid; r < nwords; r += kWarps) {
        const int i = (r << 5) + lane;
        const bool in = i < n;
        const uint32_t key = in ? get1(i) : 0u;
        const uint32_t gt = __ballot_sync(0xffffffffu, in && key > T);
        const uint32_t eq = __ballot_sync(0xffffffffu, in && key == T);
        if (lane == 0) {
            selw[r] = gt;
            tiew[r] = eq;
        }
    }
    __syncthreads();
    // each thread a run of words: counts, one 64-bit scan (ties high, keys > T low), write
    const int wpt = (nwords + kThreads - 1) / kThreads;
    const int w0 = min(tid * wpt, nwords), w1 = min(w0 + wpt, nwords);
    uint32_t cg = 0, ce = 0;
    for (int w = w0; w < w1; w++) {
        cg += __popc(selw[w]);
        ce += __popc(tiew[w]);
    }
    unsigned long long tot;
    const unsigned long long pre =
        block_exclusive_scan64(((unsigned long long)ce << 32) | cg, sh.scan64, tot);
    uint32_t ties = (uint32_t)(pre >> 32);
    uint32_t pos = (uint32_t)pre + min(ties, krem);
    for (int w = w0; w < w1; w++) {
        uint32_t take = selw[w];
        uint32_t tw = tiew[w];
        // the lowest-index ties while the budget lasts
        while (tw && ties < krem) {
            take |= tw & (0u - tw);
            tw &= tw - 1;
            ties++;
        }
        ties += __popc(tw);
        while (take) {
            const int bit = __ffs(take) - 1;
            if (pos < (uint32_t)k) out[pos] = (w << 5) + bit;
            pos++;
            take &= take - 1;
        }
    }
    // the row's total; NaN scores (no total order) break it
    if (tid == 0 && (uint32_t)tot + min((uint32_t)(tot >> 32), krem) != (uint32_t)k)
        flag(dev_status, CSA_DEV_NAN);
}

// ---- long rows: one cluster per query ------------------------------------------------
constexpr int kMaxCluster = 8;
constexpr int kClusterSlice = 32768;    // entries per rank the cluster size aims at

struct __align__(16) ClShared {
    uint32_t hist[2][kBins];   // this rank's digit histogram, double-buffered across digits
    uint32_t hsum[kBins];      // the cluster's summed histogram
    uint32_t cand[kMaxCand];   // this rank's candidates, read by the others
    uint32_t acand[kMaxCand];  // every rank's candidates, in rank order
    uint32_t scan_tmp[33];
    unsigned long long scan64[33];
    uint32_t bin, krem, ncand, above, key_or, key_and, ngt, neq, g_or, g_and, out_base, take_eq;
    uint32_t r_ncand[kMaxCluster], r_above[kMaxCluster], r_off[kMaxCluster + 1];
    uint32_t r_gt[kMaxCluster], r_eq[kMaxCluster];
};

template <bool STAGED>
__global__ void __launch_bounds__(kThreads) topk_cluster_kernel(
    const float* __restrict__ scores, int64_t ld, const int32_t* __restrict__ q_seq,
    const int32_t* __restrict__ q_pos, const int64_t* __restrict__ seq_len, int B, int m,
    int max_n, int k, int32_t* __restrict__ idx_out, int32_t* __restrict__ dev_status) {
    using namespace sm100;
    extern __shared__ uint4 dyn4[];
    ClShared& sh = *reinterpret_cast<ClShared*>(dyn4);
    const int R = (int)cluster_nctarank();
    const int rank = (int)cluster_ctarank();
    const int qq = blockIdx.x / R;
    const int tid = threadIdx.x, lane = tid & 31, wid = tid >> 5;
    const int b = q_seq[qq];
    const int t = q_pos[qq];
    const bool valid = b >= 0 && b < B && t >= 0 && (int64_t)t < seq_len[b];
    pdl_wait();   // scores come from the indexer
    pdl_trigger();
    int n = valid ? (t + 1) / m : 0;
    if (n > max_n) n = max_n;
    int32_t* out = idx_out + (int64_t)qq * k;
    if (n <= k) {
        // the same branch on every rank of the cluster: no cluster barrier is reached
        if (rank == 0)
            for (int j = tid; j < k; j += kThreads) out[j] = j < n ? j : -1;
        return;
    }
    // my slice; inner boundaries on multiples of 32 entries (whole words, 16-byte loads)
    const int lo = rank == 0 ? 0 : (int)(((int64_t)n * rank / R) & ~31LL);
    const int hi = rank == R - 1 ? n : (int)(((int64_t)n * (rank + 1) / R) & ~31LL);
    const int ns = hi - lo;
    const float* s = scores + (int64_t)qq * ld + lo;
    const bool vec = (reinterpret_cast<uintptr_t>(s) & 15) == 0;
    // after the shared state: the selection words of my slice, then its staged keys
    const int slice_max = (max_n + R - 1) / R + 32;
    const int wmax = (slice_max + 31) >> 5;
    uint32_t* selw = reinterpret_cast<uint32_t*>(&sh + 1);
    uint32_t* tiew = selw + wmax;
    uint4* skey4 = reinterpret_cast<uint4*>(selw) + ((2 * wmax + 3) >> 2);
    const uint32_t* skey = reinterpret_cast<const uint32_t*>(skey4);
    if (tid == 0) {
        sh.key_or = 0u;
        sh.key_and = 0xFFFFFFFFu;
        sh.ncand = 0u;
        sh.above = 0u;
        sh.ngt = 0u;
        sh.neq = 0u;
    }
    __syncthreads();
    auto get4 = [&](int i, uint32_t* key) {
        if constexpr (STAGED) {
            const uint4 v = i < ns ? skey4[i >> 2] : make_uint4(0u, 0u, 0u, 0u);
            key[0] = i < ns ? v.x : 0u;
            key[1] = i + 1 < ns ? v.y : 0u;
            key[2] = i + 2 < ns ? v.z : 0u;
            key[3] = i + 3 < ns ? v.w : 0u;
        } else {
            load4(s, i, ns, vec, key);
        }
    };
    auto get1 = [&](int i) -> uint32_t {
        if constexpr (STAGED) {
            return skey[i];
        } else {
            return score_key(s[i]);
        }
    };
    uint32_t kor = 0u, kand = 0xFFFFFFFFu;
    for (int c0 = 0; c0 < ns; c0 += kChunk) {
        const int i = c0 + 4 * tid;
        uint32_t key[4];
        load4(s, i, ns, vec, key);
#pragma unroll
        for (int u = 0; u < 4; u++) {
            if (i + u < ns) {
                kor |= key[u];
                kand &= key[u];
            }
        }
        if constexpr (STAGED) {
            if (i < ns) skey4[i >> 2] = make_uint4(key[0], key[1], key[2], key[3]);
        }
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
        kor |= __shfl_xor_sync(0xffffffffu, kor, o);
        kand &= __shfl_xor_sync(0xffffffffu, kand, o);
    }
    if (lane == 0) {
        atomicOr(&sh.key_or, kor);
        atomicAnd(&sh.key_and, kand);
    }
    __syncthreads();
    cluster_sync_all();   // every rank's OR / AND
    if (wid == 0) {
        uint32_t o = 0u, a = 0xFFFFFFFFu;
        if (lane < R) {
            o = ld_cluster_u32(mapa(&sh.key_or, (uint32_t)lane));
            a = ld_cluster_u32(mapa(&sh.key_and, (uint32_t)lane));
        }
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) {
            o |= __shfl_xor_sync(0xffffffffu, o, x);
            a &= __shfl_xor_sync(0xffffffffu, a, x);
        }
        if (lane == 0) {
            sh.g_or = o;
            sh.g_and = a;
        }
    }
    __syncthreads();
    const uint32_t diff = sh.g_or ^ sh.g_and;
    uint32_t prefix = sh.g_and & ~diff;
    uint32_t mask = ~diff;
    uint32_t krem = (uint32_t)k;
    int top = diff ? 31 - __clz(diff) : -1;
    int digit = 0;
    bool exchange = false;
    // cluster-wide digits on the full slices, until the chosen bin is small
    while (top >= 0) {
        const int width = top >= 10 ? 11 : top + 1;
        const int shift = top + 1 - width;
        const uint32_t bmask = (1u << width) - 1u;
        uint32_t* hist = sh.hist[digit & 1];
        for (int x = tid; x < kBins; x += kThreads) hist[x] = 0u;
        __syncthreads();
        for (int c0 = 0; c0 < ns; c0 += kChunk) {
            uint32_t key[4];
            get4(c0 + 4 * tid, key);
#pragma unroll
            for (int u = 0; u < 4; u++)
                if (c0 + 4 * tid + u < ns && (key[u] & mask) == prefix)
                    atomicAdd(&hist[(key[u] >> shift) & bmask], 1u);
        }
        __syncthreads();
        // every rank's histogram of this digit is complete (and every rank is done reading
        // the previous digit's, which this buffer's next use overwrites)
        cluster_sync_all();
        if (tid < kBins / 4) {
            uint4 acc = make_uint4(0u, 0u, 0u, 0u);
            for (int rr = 0; rr < R; rr++) {
                const uint4 v = ld_cluster_u4(mapa(hist + 4 * tid, (uint32_t)rr));
                acc.x += v.x;
                acc.y += v.y;
                acc.z += v.z;
                acc.w += v.w;
            }
            *reinterpret_cast<uint4*>(sh.hsum + 4 * tid) = acc;
        }
        __syncthreads();
        pick_bin_in(sh.hsum, sh.scan_tmp, &sh.bin, &sh.krem, krem);
        const uint32_t in_bin = sh.hsum[sh.bin];   // over the whole row: the same on every rank
        prefix |= sh.bin << shift;
        mask |= bmask << shift;
        top = shift - 1;
        digit++;
        __syncthreads();
        if (top >= 0 && in_bin <= (uint32_t)kMaxCand) {
            exchange = true;
            break;
        }
    }
    if (exchange) {
        // my keys in the chosen region become candidates; keys above it are counted
        uint32_t above = 0;
        for (int c0 = 0; c0 < ns; c0 += kChunk) {
            uint32_t key[4];
            get4(c0 + 4 * tid, key);
#pragma unroll
            for (int u = 0; u < 4; u++) {
                const bool in = c0 + 4 * tid + u < ns;
                const uint32_t mk = key[u] & mask;
                const bool p = in && mk == prefix;
                above += (in && mk > prefix) ? 1u : 0u;
                const uint32_t bal = __ballot_sync(0xffffffffu, p);
                uint32_t slot = 0;
                if (lane == 0 && bal) slot = atomicAdd(&sh.ncand, (uint32_t)__popc(bal));
                slot = __shfl_sync(0xffffffffu, slot, 0);
                if (p) sh.cand[slot + __popc(bal & lanemask_lt())] = key[u];
            }
        }
#pragma unroll
        for (int x = 16; x > 0; x >>= 1) above += __shfl_xor_sync(0xffffffffu, above, x);
        if (lane == 0) atomicAdd(&sh.above, above);
        __syncthreads();
        cluster_sync_all();   // every rank's candidates and counts
        if (wid == 0) {
            uint32_t nc = 0, ab = 0;
            if (lane < R) {
                nc = ld_cluster_u32(mapa(&sh.ncand, (uint32_t)lane));
                ab = ld_cluster_u32(mapa(&sh.above, (uint32_t)lane));
            }
            uint32_t inc = nc;
#pragma unroll
            for (int o = 1; o < 32; o <<= 1) {
                const uint32_t y = __shfl_up_sync(0xffffffffu, inc, o);
                if (lane >= o) inc += y;
            }
            if (lane < R) {
                sh.r_ncand[lane] = nc;
                sh.r_above[lane] = ab;
                sh.r_off[lane] = inc - nc;
                sh.r_gt[lane] = 0u;
                sh.r_eq[lane] = 0u;
            }
            if (lane == R - 1) sh.r_off[R] = inc;
        }
        __syncthreads();
        const uint32_t nall = sh.r_off[R];   // the chosen bin's count over the row
        for (int rr = 0; rr < R; rr++) {
            const uint32_t nc = sh.r_ncand[rr], off = sh.r_off[rr];
            for (uint32_t c = tid; c < nc; c += kThreads)
                sh.acand[off + c] = ld_cluster_u32(mapa(sh.cand + c, (uint32_t)rr));
        }
        __syncthreads();
        // the remaining bits on the full candidate list, on this rank alone
        while (top >= 0) {
            const int width = top >= 10 ? 11 : top + 1;
            const int shift = top + 1 - width;
            const uint32_t bmask = (1u << width) - 1u;
            for (int x = tid; x < kBins; x += kThreads) sh.hsum[x] = 0u;
            __syncthreads();
            for (uint32_t c = tid; c < nall; c += kThreads) {
                const uint32_t key = sh.acand[c];
                if ((key & mask) == prefix) atomicAdd(&sh.hsum[(key >> shift) & bmask], 1u);
            }
            __syncthreads();
            pick_bin_in(sh.hsum, sh.scan_tmp, &sh.bin, &sh.krem, krem);
            prefix |= sh.bin << shift;
            mask |= bmask << shift;
            top = shift - 1;
            __syncthreads();
        }
        // every rank's keys > T and == T among the candidates (runs are in rank order)
        for (uint32_t c = tid; c < nall; c += kThreads) {
            const uint32_t key = sh.acand[c];
            int rr = 0;
            while (rr + 1 < R && sh.r_off[rr + 1] <= c) rr++;
            if (key > prefix) atomicAdd(&sh.r_gt[rr], 1u);
            if (key == prefix) atomicAdd(&sh.r_eq[rr], 1u);
        }
        __syncthreads();
        if (tid == 0) {
            uint32_t g = 0, e = 0;
            for (int rr = 0; rr < rank; rr++) {
                g += sh.r_above[rr] + sh.r_gt[rr];
                e += sh.r_eq[rr];
            }
            sh.out_base = g + min(e, krem);
            sh.take_eq = min(sh.r_eq[rank], krem - min(e, krem));
        }
        __syncthreads();
    }
    const uint32_t T = prefix;   // the k-th largest key of the row
    // marking: word r holds my entries 32 r .. 32 r + 31 (bit = lane)
    const int nwords = (ns + 31) >> 5;
    for (int r = wid; r < nwords; r += kWarps) {
        const int i = (r << 5) + lane;
        const bool in = i < ns;
        const uint32_t key = in ? get1(i) : 0u;
        const uint32_t gt = __ballot_sync(0xffffffffu, in && key > T);
        const uint32_t eq = __ballot_sync(0xffffffffu, in && key == T);
        if (lane == 0) {
            selw[r] = gt;
            tiew[r] = eq;
        }
    }
    __syncthreads();
    const int wpt = (nwords + kThreads - 1) / kThreads;
    const int w0 = min(tid * wpt, nwords), w1 = min(w0 + wpt, nwords);
    uint32_t cg = 0, ce = 0;
    for (int w = w0; w < w1; w++) {
        cg += __popc(selw[w]);
        ce += __popc(tiew[w]);
    }
    unsigned long long tot;
    const unsigned long long pre =
        block_exclusive_scan64(((unsigned long long)ce << 32) | cg, sh.scan64, tot);
    if (!exchange) {
        // every bit was resolved cluster-wide: exchange the counts at T
        if (tid == 0) {
            sh.ngt = (uint32_t)tot;
            sh.neq = (uint32_t)(tot >> 32);
        }
        __syncthreads();
        cluster_sync_all();   // every rank's counts
        if (wid == 0) {
            uint32_t g = 0u, e = 0u;
            if (lane < rank) {
                g = ld_cluster_u32(mapa(&sh.ngt, (uint32_t)lane));
                e = ld_cluster_u32(mapa(&sh.neq, (uint32_t)lane));
            }
#pragma unroll
            for (int x = 16; x > 0; x >>= 1) {
                g += __shfl_xor_sync(0xffffffffu, g, x);
                e += __shfl_xor_sync(0xffffffffu, e, x);
            }
            if (lane == 0) {
                sh.out_base = g + min(e, krem);
                sh.take_eq = min(sh.neq, krem - min(e, krem));
            }
        }
        __syncthreads();
    }
    const uint32_t budget = sh.take_eq;
    uint32_t ties = (uint32_t)(pre >> 32);
    uint32_t pos = sh.out_base + (uint32_t)pre + min(ties, budget);
    for (int w = w0; w < w1; w++) {
        uint32_t take = selw[w];
        uint32_t tw = tiew[w];
        while (tw && ties < budget) {
            take |= tw & (0u - tw);
            tw &= tw - 1;
            ties++;
        }
        ties += __popc(tw);
        while (take) {
            const int bit = __ffs(take) - 1;
            if (pos < (uint32_t)k) out[pos] = lo + (w << 5) + bit;
            pos++;
            take &= take - 1;
        }
    }
    // the last rank ends at the row's total; NaN scores (no total order) break it
    if (tid == 0 && rank == R - 1 &&
        sh.out_base + (uint32_t)tot + min((uint32_t)(tot >> 32), budget) != (uint32_t)k)
        flag(dev_status, CSA_DEV_NAN);
    // no rank leaves while another may still read its shared memory
    cluster_sync_all();
}

}  // namespace

cudaError_t launch_topk(const float* scores, int64_t ld, const int32_t* q_seq,
                        const int32_t* q_pos, const int64_t* seq_len, int Q, int B, int m,
                        int max_n, int k, int32_t* idx_out, int32_t* st, cudaStream_t stream,
                        const uint32_t* gmax, int64_t ld_g) {
    if (Q == 0) return cudaSuccess;
    // rows of up to ~44K scores are staged in shared memory as keys (with the ~25 KB of
    // histogram and candidate space this stays under the 227 KB per-CTA limit)
    const size_t row_bytes = (size_t)((max_n + 3) / 4) * 16;
    const size_t word_bytes = (size_t)((2 * ((max_n + 31) / 32) + 3) / 4) * 16;
    const bool staged = word_bytes + row_bytes <= (size_t)176 * 1024;
    cudaError_t e;
    // With the indexer's group maxima every row takes one CTA: the group path reads about
    // k groups of the row; only a query whose bound admits more than cap entries falls back
    // to its full row in the same CTA (staged in shared memory when it fits).
    const int cap = 4 * k;
    const size_t gbytes = group_smem_bytes(max_n, cap);
    if (gmax && gbytes <= (size_t)176 * 1024) {
        const size_t sm = std::max(staged ? word_bytes + row_bytes : word_bytes, gbytes);
        auto kernel = staged ? topk_radix_kernel<true> : topk_radix_kernel<false>;
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)sm);
        if (e != cudaSuccess) return e;
        LaunchScope scope(kKTopk, stream);
        return launch_pdl(kernel, dim3(Q), dim3(kThreads), sm, stream, scores, ld, q_seq, q_pos,
                          seq_len, B, m, max_n, k, idx_out, st, gmax, ld_g, cap);
    }
    if (staged) {
        const size_t smem = word_bytes + row_bytes;
        e = cudaFuncSetAttribute(topk_radix_kernel<true>,
                                 cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
        if (e != cudaSuccess) return e;
        LaunchScope scope(kKTopk, stream);
        return launch_pdl(topk_radix_kernel<true>, dim3(Q), dim3(kThreads), smem, stream, scores,
                          ld, q_seq, q_pos, seq_len, B, m, max_n, k, idx_out, st,
                          (const uint32_t*)nullptr, (int64_t)0, 0);
    }
    // long rows: a cluster of R CTAs per query, about kClusterSlice entries each (the
    // selected set is unique under the total order, so the split does not change it)
    int R = (max_n + kClusterSlice - 1) / kClusterSlice;
    R = R < 2 ? 2 : (R > kMaxCluster ? kMaxCluster : R);
    const int slice_max = (max_n + R - 1) / R + 32;
    const int wmax = (slice_max + 31) / 32;
    const size_t cl_words = (size_t)((2 * wmax + 3) / 4) * 16;
    const size_t cl_row = (size_t)((slice_max + 3) / 4) * 16;
    static_assert(sizeof(ClShared) % 16 == 0, "the words follow the shared state");
    const bool cl_staged = sizeof(ClShared) + cl_words + cl_row <= (size_t)220 * 1024;
    const size_t smem = sizeof(ClShared) + cl_words + (cl_staged ? cl_row : 0);
    auto kernel = cl_staged ? topk_cluster_kernel<true> : topk_cluster_kernel<false>;
    e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    LaunchScope scope(kKTopk, stream);
    return launch_pdl_cluster(kernel, dim3(Q * R), dim3(kThreads), smem, stream, R, scores, ld,
                              q_seq, q_pos, seq_len, B, m, max_n, k, idx_out, st);
}

}  // namespace csa
