// Steps a5/a6 on the 5th-generation tensor cores: shared-KV MQA over compressed entries
// plus the sliding window, with the attention sink and partial / inverse RoPE
// ("DeepSeek-V4 深度分析报告" 2.1 CSA / HCA and "其他注意力技术细节").  Shape: 64 query
// heads, head dim 128, bf16 entries.
//
// The keys of a query form a list of 128-key tiles: tile 0 is the window (its raw rows
// RMSNormed and RoPEd here, one row per thread), tiles 1.. are the selected entries
// (sparse, gathered by index) or all visible entries (dense, contiguous).  A work item is
// (query, chunk of tiles); a chunk ends as an fp32 partial softmax state (running max, sum,
// unnormalised output) per head.  Sparse attention runs one thread-block cluster per query:
// rank 0 takes the window tile, ranks 1.. split the selected-entry tiles; each rank then
// stores its partial state of every head straight into the shared memory of the rank that
// finishes that head (posted distributed-shared-memory stores), and each rank combines its
// slice of the heads locally (ranks in order, the sink first).  Dense attention splits every
// query into the window tile and fixed 8-tile chunks of entries, whose partial states a
// second kernel combines in chunk order.  Both splits depend only on k or on the query's own length, never on the batch,
// so both paths are batch-invariant.
//
// Roles per CTA (11 warps, persistent over items):
//   warp 0      producer: dense tiles by two 2D TMA loads (64 channels x 128 rows each,
//               128-byte swizzle), sparse tiles by TMA tile::gather4 loads of the selected
//               rows (4 rows x 64 channels each; an invalid index is row -1, zero-filled) into
//               the same swizzled layout; a per-tile validity mask; 3-stage ring.
//   warp 1      TMEM allocation; lane 0 issues tcgen05.mma kind::f16 S = Q K^T as two
//               M=64 x N=64 halves (keys 0-63 -> TMEM lanes 0-15 of each quarter, keys
//               64-127 -> lanes 16-31).
//   warp 10     lane 0 issues P V, accumulated in TMEM as two outputs O_0 / O_1 (the key
//               column-halves below), each two M=64 x N=64 halves (channels 0-63 / 64-127),
//               V being the key tile read MN-major.
//   warps 2-9   two warps per TMEM lane quarter.  Per item: q heads RoPEd at t and the
//               window tile into shared memory (all 256 threads).  Per tile: 32 keys of one
//               head per thread from TMEM, softmax in the log2 domain against a reference
//               maximum that moves only on a jump of more than 2^8 (then O_ch is rescaled in
//               TMEM), P as bf16 into shared memory.  Per item: O_0 and O_1 merged, then the
//               partial state combined across the cluster (sparse) or written for the
//               combine kernel.
// All waits are bounded (timeout -> CSA_DEV_TIMEOUT, drain, free TMEM, return).
#include <cstring>
#include <mutex>

#include "launchers.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kH = 64;
constexpr int kD = 128;
constexpr int kTK = 128;                     // keys per tile
constexpr int kStages = 3;
constexpr int kBlk = kTK * 128;              // one 64-channel slice of a key tile (16 KB)
constexpr int kTileBytes = 2 * kBlk;         // 32 KB
constexpr int kQBlk = kH * 128;              // one 64-channel slice of Q (8 KB)
constexpr int kPBlk = kH * 128;              // one 64-key slice of P (8 KB)
constexpr int kThreads = 352;
static_assert(kTK / 4 == 32, "one 4-row gather group per producer lane");
constexpr int kPvWarp = 10;                  // the P V issuer
constexpr float kRescale = 8.f;              // a tile moves the reference maximum only when
                                             // it exceeds it by more than 2^8
constexpr int kDenseChunkTiles = 8;
constexpr int kMaxK = 2048;
constexpr int kMaxCluster = 8;
// sparse receive buffer: C ranks x ceil(kH / C) heads x (kD + 2) floats, largest over C >= 1
constexpr int recv_floats(int C) {
    return C > kMaxCluster ? 0
                           : (C * ((kH + C - 1) / C) * (kD + 2) > recv_floats(C + 1)
                                  ? C * ((kH + C - 1) / C) * (kD + 2)
                                  : recv_floats(C + 1));
}
constexpr int kRecvFloats = recv_floats(1);
// combine weights [heads a rank finishes][kMaxCluster + 1]: all kH heads for a cluster of one
constexpr int kWtabFloats = kH * (kMaxCluster + 1);
// a rank of a C-CTA cluster finishes at most ceil(kH / C) heads, each with kMaxCluster + 1
// weights: the table must hold that for every cluster size the launcher may pick
constexpr bool wtab_fits(int C) {
    return C > kMaxCluster ||
           ((kH + C - 1) / C * (kMaxCluster + 1) <= kWtabFloats && wtab_fits(C + 1));
}
static_assert(wtab_fits(1), "combine-weight table too small for some cluster size");
constexpr float kLog2e = 1.4426950408889634f;

struct AttnTcArgs {
    const uint16_t* q;
    const uint8_t* entries;
    EntryRows er;
    const uint16_t* kv;
    RawRows raw;
    const int32_t* q_seq;
    const int32_t* q_pos;
    const int64_t* seq_len;
    const int32_t* idx;   // nullptr: dense
    const float* sink;
    uint16_t* out;
    float* part;          // dense partials [items][kH][kD + 2]
    int32_t* st;
    int64_t ent_rows;
    int k, m, B, W, Q, chunk_tiles, chunks_per_q, total_items, max_n;
    int cluster;          // sparse: CTAs per query (one cluster); dense: 1
    // dense only: 0 = the chunks of a query spread over CTAs, combined by
    // attn_combine_kernel; 1 = one CTA takes all chunks of a query and combines them itself
    int single;
    int hreal;            // query heads of the call (16 or 64): heads >= hreal are zero padding
    float scale_log2;
    float eps;
    double log2_theta;
};

struct AItem {
    int q, b, t, c;
    int n_vis;      // visible entries
    int n_ent;      // entries in the key list (k for sparse, n_vis for dense)
    int w0, n_win;
    int tile0, ntiles;
    int64_t row0;
};

__device__ __forceinline__ bool get_item(const AttnTcArgs& a, int it, AItem& x, bool report) {
    x.q = it / a.chunks_per_q;
    x.c = it - x.q * a.chunks_per_q;
    x.b = a.q_seq[x.q];
    x.t = a.q_pos[x.q];
    if (x.b < 0 || x.b >= a.B || x.t < 0 || (int64_t)x.t >= a.seq_len[x.b]) {
        if (report && x.c == 0) flag(a.st, CSA_DEV_OOB);
        return false;
    }
    x.n_vis = (x.t + 1) / a.m;
    x.row0 = a.er.bt ? 0 : a.er.ent_off[x.b];   // dense reads contiguous rows only
    if (a.idx) {
        x.n_ent = a.k;
    } else {
        int n = x.n_vis;
        if (n > a.max_n) {
            if (report && x.c == 0) flag(a.st, CSA_DEV_CAPACITY);
            n = a.max_n;
        }
        const int64_t avail = a.ent_rows - x.row0;
        if ((int64_t)n > avail) {
            if (report && x.c == 0) flag(a.st, CSA_DEV_OOB);
            n = avail > 0 ? (int)avail : 0;
        }
        x.n_ent = n;
    }
    x.w0 = x.t - a.W + 1 > 0 ? x.t - a.W + 1 : 0;
    x.n_win = a.W > 0 ? x.t - x.w0 + 1 : 0;
    const int n_et = (x.n_ent + kTK - 1) / kTK;   // entry tiles
    if (a.idx) {
        // sparse: a cluster of one CTA takes every tile; in a larger cluster rank 0 takes
        // the window tile and ranks 1..C-1 split the entry tiles contiguously (the host
        // picks C - 1 <= n_et: every rank has one)
        const int C = a.cluster;
        if (C == 1) {
            x.tile0 = 0;
            x.ntiles = 1 + n_et;
        } else if (x.c == 0) {
            x.tile0 = 0;
            x.ntiles = 1;
        } else {
            const int lo = 1 + (x.c - 1) * n_et / (C - 1), hi = 1 + x.c * n_et / (C - 1);
            x.tile0 = lo;
            x.ntiles = hi - lo;
        }
        return x.ntiles > 0;
    }
    // dense: chunk 0 is the window tile alone (its rows are built in-kernel, which takes as
    // long as several entry tiles), chunks 1.. take chunk_tiles entry tiles each
    if (x.c == 0) {
        x.tile0 = 0;
        x.ntiles = 1;
    } else {
        x.tile0 = 1 + (x.c - 1) * a.chunk_tiles;
        x.ntiles = min(a.chunk_tiles, 1 + n_et - x.tile0);
    }
    return x.ntiles > 0;
}

// The i-th item this CTA takes, or -1 past its last.  Spread (dense chunks and sparse
// queries): items blockIdx.x, blockIdx.x + gridDim.x, ...  Single (dense): every chunk of
// queries blockIdx.x, blockIdx.x + gridDim.x, ..., a query's chunks in order.
__device__ __forceinline__ int item_id(const AttnTcArgs& a, int i) {
    if (!a.single) {
        const int it = (int)blockIdx.x + i * (int)gridDim.x;
        return it < a.total_items ? it : -1;
    }
    const int q = (int)blockIdx.x + (i / a.chunks_per_q) * (int)gridDim.x;
    return q < a.Q ? q * a.chunks_per_q + i % a.chunks_per_q : -1;
}

// Chunks of a dense query: the window chunk, then its entry tiles in chunks of
// chunk_tiles (a function of the query's own visible entries).
__device__ __forceinline__ int dense_chunks(const AttnTcArgs& a, int q, int& t) {
    const int b = a.q_seq[q];
    t = a.q_pos[q];
    if (b < 0 || b >= a.B || t < 0 || (int64_t)t >= a.seq_len[b]) return 0;
    int n = (t + 1) / a.m;
    if (n > a.max_n) n = a.max_n;
    const int64_t avail = a.ent_rows - a.er.ent_off[b];
    if ((int64_t)n > avail) n = avail > 0 ? (int)avail : 0;
    return 1 + ((n + kTK - 1) / kTK + a.chunk_tiles - 1) / a.chunk_tiles;
}

// The output of channels d, d + 1 (d even) of head h of dense query q at position t: the
// nch chunk partials combined in chunk order with the sink first (M = max(sink, m_c),
// w_c = 2^(m_c - M), L = 2^(sink - M) + sum_c w_c l_c, o = sum_c w_c O_c / L), then the
// inverse RoPE on the last 64 channels.  Both dense variants combine with this function, so
// a query's bits do not depend on which one ran.
__device__ __forceinline__ float2 combine_pair(const AttnTcArgs& a, int q, int t, int nch,
                                               int h, int d) {
    const float* base = a.part + ((int64_t)q * a.chunks_per_q * kH + h) * (kD + 2);
    const int64_t cstride = (int64_t)kH * (kD + 2);
    const float sk = a.sink[h] * kLog2e;
    float M = sk;
    for (int c = 0; c < nch; c++) M = fmaxf(M, base[c * cstride]);
    float L = (M == -INFINITY || sk == -INFINITY) ? 0.f : exp2f(sk - M);
    float o0 = 0.f, o1 = 0.f;
    for (int c = 0; c < nch; c++) {
        const float* pc = base + c * cstride;
        const float mc = pc[0];
        const float w = (mc == -INFINITY) ? 0.f : exp2f(mc - M);
        L = fmaf(w, pc[1], L);
        const float2 v = *reinterpret_cast<const float2*>(pc + 2 + d);
        o0 = fmaf(w, v.x, o0);
        o1 = fmaf(w, v.y, o1);
    }
    o0 = L > 0.f ? o0 / L : 0.f;
    o1 = L > 0.f ? o1 / L : 0.f;
    if (d >= kD - kRopeDims) {
        float cs, sn;   // rotation by -t
        rope_cos_sin(-(double)t, (d - (kD - kRopeDims)) >> 1, a.log2_theta, cs, sn);
        const float x = o0, y = o1;
        o0 = x * cs - y * sn;
        o1 = x * sn + y * cs;
    }
    return make_float2(o0, o1);
}

// Byte offset of 16-byte chunk `ch` of row `r` in a 128-byte-swizzled [rows x 128 B] block.
__device__ __forceinline__ uint32_t swz(int r, int ch) {
    return (uint32_t)(r * 128 + ((ch ^ (r & 7)) << 4));
}

__device__ __forceinline__ void fence_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// MN-major 128-byte-swizzled operand descriptor (rows of 128 B along MN, 8-row groups
// 1024 B apart along K; LBO = distance between 64-element MN slices).
__device__ __forceinline__ uint64_t smem_desc_mn_sw128(const void* tile, uint32_t lbo_bytes) {
    const uint64_t addr = sm100::smem_addr(tile);
    uint64_t d = 0;
    d |= (addr >> 4) & 0x3FFFull;
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)(1024 >> 4) << 32;
    d |= 1ull << 46;
    d |= 2ull << 61;
    return d;
}

__global__ void __launch_bounds__(kThreads, 1)
    attn_tc_kernel(const __grid_constant__ CUtensorMap tmap_e,
                   const __grid_constant__ CUtensorMap tmap_g, const AttnTcArgs a) {
    using namespace sm100;
    constexpr uint32_t kIdescS = instr_desc(1, 1, 64, 64);
    constexpr uint32_t kIdescPV = instr_desc(1, 1, 64, 64, 1);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sK = smem;                              // [kStages][2][128 x 128 B]
    uint8_t* sW = sK + kStages * kTileBytes;         // window tile [2][128 x 128 B]
    uint8_t* sQ = sW + kTileBytes;                   // [2][64 x 128 B]
    uint8_t* sP = sQ + 2 * kQBlk;                    // [2 buffers][2][64 x 128 B]
    uint32_t* smask = reinterpret_cast<uint32_t*>(sP + 4 * kPBlk);   // [kStages + 1][4]
    // per item RoPE tables, pair j of the last 64 dims: frequency, cos/sin at t, and
    // cos/sin at the window's first position
    float* rf = reinterpret_cast<float*>(smask + 4 * (kStages + 1));  // [32]
    float* rqc = rf + 32;
    float* rqs = rqc + 32;
    float* rwc = rqs + 32;
    float* rws = rwc + 32;
    int32_t* sidx = reinterpret_cast<int32_t*>(rws + 32);   // [kMaxK] the item's index row
    int32_t* srows = sidx + kMaxK;                          // [kStages][128] gather rows
    // sparse: receive buffer of the partial states of this rank's heads from every rank,
    // [cluster][nh][kD] O then [cluster][2][nh] m, l (nh = heads per rank); then the
    // per-head combine weights [nh][kMaxCluster + 1], nh <= kH
    float* recv = reinterpret_cast<float*>(srows + kStages * kTK);
    float* wtab = recv + kRecvFloats;
    float* xml = wtab + kWtabFloats;       // [128][2] column-half 1's m, l per (head, half)
    uint64_t* bars = reinterpret_cast<uint64_t*>(xml + 256);
    uint64_t* full = bars;                 // [kStages]  33 arrivals (+tx)
    uint64_t* empty = full + kStages;      // [kStages]  MMA commit
    uint64_t* prep_full = empty + kStages; // Q + window ready: 8 arrivals
    uint64_t* prep_empty = prep_full + 1;  // item's MMAs done: MMA commit
    uint64_t* s_full = prep_empty + 1;     // [2]
    uint64_t* s_empty = s_full + 2;        // [2] 8 arrivals
    uint64_t* p_full = s_empty + 2;        // [2] 8 arrivals
    uint64_t* p_empty = p_full + 2;        // [2]
    uint64_t* pvdone = p_empty + 2;        // MMA commit after every tile's P V (a rescale
                                           // waits for the previous one)
    uint64_t* odone = pvdone + 1;          // MMA commit after an item's last P V
    uint64_t* cpart_full = odone + 3;     // every rank's partials are in: 4 x cluster
    uint64_t* cpart_free = cpart_full + 1; // every rank has combined the previous query (its
                                           // receive buffer is free again): 4 x cluster
    uint64_t* drain = cpart_free + 1;
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full[s], 33);
            mbar_init(&empty[s], 1);
        }
        mbar_init(prep_full, 8);
        mbar_init(prep_empty, 1);
        for (int i = 0; i < 2; i++) {
            mbar_init(&s_full[i], 1);
            mbar_init(&s_empty[i], 8);
            mbar_init(&p_full[i], 8);
            mbar_init(&p_empty[i], 1);
        }
        mbar_init(pvdone, 1);
        mbar_init(odone, 1);
        mbar_init(cpart_full, 4 * a.cluster);
        mbar_init(cpart_free, 4 * a.cluster);
        mbar_init(drain, 2);   // both MMA issuers
        *abort_flag = 0;
        mbar_fence_init();
        prefetch_tmap(a.idx ? &tmap_g : &tmap_e);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, 256);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    // the cluster's barriers are initialised before any rank arrives on another's
    if (a.cluster > 1) cluster_sync_all();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_smem;
    const uint32_t tmem_S = tmem_base;          // [2] x 64 columns
    const uint32_t tmem_O = tmem_base + 128;    // O_0, O_1: 64 columns each

    if (warp == 0) {
        // ---------------- producer ----------------
        // index sets (top-k) and entries (compression) come from earlier kernels; the
        // prologue of the other roles (q heads, window rows) only reads inputs
        int stage = 0;
        uint32_t ph = 0;
        int issued[kStages] = {};
        bool ok = true;
        bool waited = false;
        for (int ii = 0; ok; ii++) {
            const int it = item_id(a, ii);
            if (it < 0) break;
            AItem x;
            const bool have = get_item(a, it, x, false);
            if (have && !a.idx) {
                // dense: the item's entry tiles are contiguous rows; all of them are
                // prefetched into L2 at once (before the wait on the previous kernel for the
                // first item: a prefetch returns no data, and L2 holds the coherent copy of
                // the entries the previous kernel writes), so the tile loads below meet L2
                for (int jj = lane; jj < x.ntiles; jj += 32) {
                    const int j = x.tile0 + jj;
                    const int e0 = (j - 1) * kTK;
                    const int rows = j == 0 ? 0 : min(kTK, x.n_ent - e0);
                    if (rows > 0)
                        prefetch_l2_bulk(a.entries + (x.row0 + e0) * (int64_t)(kD * 2),
                                         (uint32_t)(rows * kD * 2));
                }
            }
            if (!waited) {
                pdl_wait();
                if (lane == 0) pdl_trigger();
                waited = true;
            }
            if (!have) continue;
            if (a.idx && x.tile0 + x.ntiles > 1) {
                // the query's whole index row, once per item: batches of 8 x 16-byte loads
                // per lane in flight (one round trip for k <= 1024); only this warp reads it
                const int32_t* src = a.idx + (int64_t)x.q * a.k;
                if ((a.k & 3) == 0 && (reinterpret_cast<uintptr_t>(src) & 15) == 0) {
                    const int n4 = a.k >> 2;
                    for (int base = 0; base < n4; base += 32 * 8) {
                        int4 v[8];
#pragma unroll
                        for (int u = 0; u < 8; u++) {
                            const int j4 = base + lane + 32 * u;
                            if (j4 < n4) v[u] = *reinterpret_cast<const int4*>(src + 4 * j4);
                        }
#pragma unroll
                        for (int u = 0; u < 8; u++) {
                            const int j4 = base + lane + 32 * u;
                            if (j4 < n4) *reinterpret_cast<int4*>(sidx + 4 * j4) = v[u];
                        }
                    }
                } else {
                    for (int base = 0; base < a.k; base += 32 * 8) {
                        int v[8];
#pragma unroll
                        for (int u = 0; u < 8; u++) {
                            const int j = base + lane + 32 * u;
                            v[u] = j < a.k ? src[j] : -1;
                        }
#pragma unroll
                        for (int u = 0; u < 8; u++) {
                            const int j = base + lane + 32 * u;
                            if (j < a.k) sidx[j] = v[u];
                        }
                    }
                }
                __syncwarp();
            }
            for (int jj = 0; jj < x.ntiles; jj++) {
                const int j = x.tile0 + jj;
                if (j == 0) continue;  // the window tile is built by the softmax warps
                if (!mbar_wait_warp(&empty[stage], ph ^ 1, abort_flag, a.st)) {
                    ok = false;
                    break;
                }
                uint8_t* dst = sK + stage * kTileBytes;
                const int e0 = (j - 1) * kTK;
                if (!a.idx) {
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[stage], kTileBytes);
                        tma_load_2d(dst, &tmap_e, &full[stage], 0, (int32_t)(x.row0 + e0));
                        tma_load_2d(dst + kBlk, &tmap_e, &full[stage], 64, (int32_t)(x.row0 + e0));
                    }
#pragma unroll
                    for (int rr = 0; rr < 4; rr++) {
                        const unsigned v = __ballot_sync(0xffffffffu, e0 + lane + 32 * rr < x.n_ent);
                        if (lane == 0) smask[stage * 4 + rr] = v;
                    }
                    __syncwarp();
                    if (lane != 0) mbar_arrive(&full[stage]);
                } else {
                    // rows of the selected entries: lanes resolve 4 each (invalid -> row -1,
                    // which the TMA zero-fills), lane 0 issues 4-row gathers per 64 channels
                    int32_t* rows = srows + stage * kTK;
#pragma unroll
                    for (int rr = 0; rr < 4; rr++) {
                        const int r = lane + 32 * rr;
                        const int v = e0 + r;
                        int32_t row = -1;
                        if (v < x.n_ent) {
                            const int e = sidx[v];
                            if (e >= 0) {
                                const int64_t re = a.er.bt ? a.er.row(x.b, e) : x.row0 + e;
                                if (e < x.n_vis && re >= 0 && re < a.ent_rows) {
                                    row = (int32_t)re;
                                } else {
                                    flag(a.st, CSA_DEV_OOB);
                                }
                            }
                        }
                        rows[r] = row;
                        const unsigned vm = __ballot_sync(0xffffffffu, row >= 0);
                        if (lane == 0) smask[stage * 4 + rr] = vm;
                    }
                    // the tile's byte count is expected before any gather is issued; then every
                    // lane issues the two gathers (both channel halves) of its own 4-row group,
                    // since one thread issuing all 64 would serialise on the issue cost
                    if (lane == 0) mbar_arrive_expect_tx(&full[stage], kTileBytes);
                    __syncwarp();
                    {
                        const int g = lane;   // kTK / 4 = 32 row groups
                        const int32_t r0 = rows[4 * g], r1 = rows[4 * g + 1], r2 = rows[4 * g + 2],
                                      r3 = rows[4 * g + 3];
                        tma_gather4(dst + 4 * g * 128, &tmap_g, &full[stage], 0, r0, r1, r2, r3);
                        tma_gather4(dst + kBlk + 4 * g * 128, &tmap_g, &full[stage], 64, r0, r1, r2, r3);
                    }
                    if (lane != 0) mbar_arrive(&full[stage]);
                }
                if (lane == 0) mbar_arrive(&full[stage]);
                issued[stage]++;
                if (++stage == kStages) {
                    stage = 0;
                    ph ^= 1;
                }
            }
        }
        if (!waited) {
            pdl_wait();
            if (lane == 0) pdl_trigger();
        }
        for (int s = 0; s < kStages; s++)
            if (issued[s]) mbar_drain(&full[s], (issued[s] - 1) & 1, a.st);
    } else if (warp == 1 || warp == kPvWarp) {
        if (lane == 0) {
            // ---------------- MMA issuers ----------------
            // One tcgen05.mma costs its issuing thread tens of cycles however small it is, so
            // the small MMAs here are issued by two threads: warp 1 issues S = Q K^T of every
            // tile (as soon as its keys and an S buffer are there), warp kPvWarp issues P V.
            // P V accumulates into the item's two running outputs in TMEM, one per key
            // column-half: O_0 takes keys 0-31 and 64-95 of every tile (K-steps 0, 1, 4, 5),
            // O_1 keys 32-63 and 96-127.  P of a tile being ready implies its S was consumed,
            // so the P V issuer follows the key ring without waiting on the loads, and its
            // commits alone release key stages, P buffers and the item.
            const bool s_role = warp == 1;
            int stage = 0;
            uint32_t ph = 0;
            int nt = 0, nitem = 0;
            bool ok = true;
            for (int ii = 0; ok; ii++) {
                const int it = item_id(a, ii);
                if (it < 0) break;
                AItem x;
                if (!get_item(a, it, x, false)) continue;
                if (s_role) {
                    if (!mbar_wait(prep_full, nitem & 1, abort_flag, a.st)) break;
                    fence_async_smem();
                    tc_fence_after();
                }
                for (int jj = 0; jj < x.ntiles && ok; jj++) {
                    const int j = x.tile0 + jj;
                    const uint8_t* kb;
                    int my_stage = -1;
                    if (j == 0) {
                        kb = sW;
                    } else {
                        if (s_role && !mbar_wait(&full[stage], ph, abort_flag, a.st)) {
                            ok = false;
                            break;
                        }
                        kb = sK + stage * kTileBytes;
                        my_stage = stage;
                        if (++stage == kStages) {
                            stage = 0;
                            ph ^= 1;
                        }
                    }
                    const int sb = nt & 1;
                    if (s_role) {
                        if (!mbar_wait(&s_empty[sb], ((nt >> 1) & 1) ^ 1, abort_flag, a.st)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
                        // the two key halves are independent accumulators: interleave their chains
#pragma unroll
                        for (int kk = 0; kk < 8; kk++) {
#pragma unroll
                            for (int half = 0; half < 2; half++) {
                                const uint32_t d = tmem_S + sb * 64 + ((uint32_t)(half * 16) << 16);
                                const int blk = kk >> 2;
                                const uint32_t off = (uint32_t)((kk & 3) * 32) >> 4;
                                const uint64_t ad = smem_desc_k_sw128(sQ + blk * kQBlk) + off;
                                const uint64_t bd =
                                    smem_desc_k_sw128(kb + blk * kBlk + half * 64 * 128) + off;
                                mma_f16(d, ad, bd, kIdescS, kk > 0 ? 1u : 0u);
                            }
                        }
                        mma_commit(&s_full[sb]);
                    } else {
                        if (!mbar_wait(&p_full[sb], (nt >> 1) & 1, abort_flag, a.st)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll
                        for (int ch = 0; ch < 2; ch++) {
#pragma unroll
                            for (int t = 0; t < 4; t++) {
                                const int kk = (t >> 1) * 4 + ch * 2 + (t & 1);
                                const uint64_t ad =
                                    smem_desc_k_sw128(sP + sb * 2 * kPBlk + (kk >> 2) * kPBlk) +
                                    ((uint32_t)((kk & 3) * 32) >> 4);
#pragma unroll
                                for (int half = 0; half < 2; half++) {
                                    const uint32_t d = tmem_O + ch * 64 + ((uint32_t)(half * 16) << 16);
                                    const uint64_t bd =
                                        smem_desc_mn_sw128(kb + half * kBlk + kk * 2048, kBlk);
                                    mma_f16(d, ad, bd, kIdescPV, (jj == 0 && t == 0) ? 0u : 1u);
                                }
                            }
                        }
                        mma_commit(&p_empty[sb]);
                        if (my_stage >= 0) mma_commit(&empty[my_stage]);
                        mma_commit(pvdone);
                    }
                    nt++;
                }
                if (!ok) break;
                if (!s_role) {
                    mma_commit(odone);
                    mma_commit(prep_empty);
                }
                nitem++;
            }
            mma_commit(drain);
            mbar_drain(drain, 0, a.st);
        }
    } else if (warp >= 2 && warp < 10) {
        // ---------------- softmax / epilogue (warps 2..9) ----------------
        // Two warps share each TMEM lane quarter (the quarter is fixed by the warp's rank
        // modulo 4): warp column-half `ch` reads S columns ch*32 .. ch*32+31 of its lanes, so a
        // thread holds 32 keys of one head (lanes 0-15: keys ch*32 + c, lanes 16-31: keys
        // 64 + ch*32 + c).  Each (head, column-half) keeps its own running maximum, sum and
        // output O_ch; the two are merged once per item.
        const int quarter = warp & 3;
        const int ch = (warp - 2) >> 2;
        const int i = threadIdx.x - 64;         // 0..255
        const int h = quarter * 16 + (lane & 15);
        const int kh = lane >> 4;               // key half of S / channel half of O
        const uint32_t lane_base = (uint32_t)(quarter * 32) << 16;
        bool waited_prev = false;
        int nt = 0, nitem = 0;
        int kst = 0;   // ring position of the next entry tile (mirrors the producer)
        bool ok = true;
        // single dense variant: after the last chunk of each query, its combine (all 256
        // threads, the query's partials written by this CTA before the barrier)
        auto combine_here = [&](int it) {
            if (!a.single || it % a.chunks_per_q != a.chunks_per_q - 1) return;
            asm volatile("bar.sync 1, 256;" ::: "memory");
            const int q = it / a.chunks_per_q;
            int t;
            const int nch = dense_chunks(a, q, t);
            if (nch == 0) return;
            if (!waited_prev) {
                pdl_wait();
                waited_prev = true;
            }
            for (int u = i; u < a.hreal * (kD / 2); u += 256) {
                const int hh = u / (kD / 2), d = 2 * (u % (kD / 2));
                const float2 o = combine_pair(a, q, t, nch, hh, d);
                *reinterpret_cast<uint32_t*>(a.out + ((int64_t)q * a.hreal + hh) * kD + d) = pack_bf16x2(o.x, o.y);
            }
        };
        for (int ii = 0;; ii++) {
            const int it = item_id(a, ii);
            if (it < 0) break;
            AItem x;
            if (!get_item(a, it, x, i == 0)) {
                combine_here(it);
                continue;
            }
            // ---- item prologue: q heads and (chunk 0) the window tile ----
            // A failed wait in a warp only skips the rest of that item; here, once per item,
            // all 256 threads meet and leave together if any of them failed.
            const bool ready = ok && mbar_wait(prep_empty, (nitem & 1) ^ 1, abort_flag, a.st);
            if (!named_barrier_and(1, 256, ready)) break;
            if (i < 32) {
                // angles in fp64, reduced, then sincosf (see rope_cos_sin)
                float cs, sn;
                rope_cos_sin((double)x.t, i, a.log2_theta, cs, sn);
                rqc[i] = cs;
                rqs[i] = sn;
                rope_cos_sin((double)x.w0, i, a.log2_theta, cs, sn);
                rwc[i] = cs;
                rws[i] = sn;
                rf[i] = (float)exp2(-(double)(2 * i) * (1.0 / 64.0) * a.log2_theta);
            } else if (i < 36 && x.tile0 == 0) {
                // window validity words: rows r with r < n_win and w0 + r >= kv_pos0
                const int wd = i - 32;
                const int64_t lo64 = a.raw.first(x.b, a.seq_len[x.b]) - (int64_t)x.w0;
                const int lo = lo64 > 0 ? (lo64 > kTK ? kTK : (int)lo64) : 0;
                const int a0 = max(lo - 32 * wd, 0), a1 = min(x.n_win - 32 * wd, 32);
                uint32_t wbits = 0;
                if (a1 > a0) wbits = (a1 - a0 == 32 ? 0xffffffffu : ((1u << (a1 - a0)) - 1u)) << a0;
                smask[kStages * 4 + wd] = wbits;
            }
            asm volatile("bar.sync 1, 256;" ::: "memory");
            {
                // q head hq, channels u*32 .. u*32+31 (RoPE on the last 64: u = 2, 3)
                const int hq = i >> 2, u = i & 3;
                // heads past the call's (16-head calls padded to the 64-head tile) are zero
                const bool hv = hq < a.hreal;
                const uint16_t* src = a.q + ((int64_t)x.q * a.hreal + (hv ? hq : 0)) * kD + u * 32;
                float v[32];
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    const uint4 w = hv ? *reinterpret_cast<const uint4*>(src + 8 * c)
                                       : make_uint4(0u, 0u, 0u, 0u);
                    const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                    for (int z = 0; z < 4; z++) {
                        const float2 f = bf16x2_to_f32(w4[z]);
                        v[8 * c + 2 * z] = f.x;
                        v[8 * c + 2 * z + 1] = f.y;
                    }
                }
                if (u >= 2) {
#pragma unroll
                    for (int k = 0; k < 16; k++) {
                        const int pj = (u - 2) * 16 + k;
                        const float cs = rqc[pj], sn = rqs[pj];
                        const float x0 = v[2 * k], y0 = v[2 * k + 1];
                        v[2 * k] = x0 * cs - y0 * sn;
                        v[2 * k + 1] = x0 * sn + y0 * cs;
                    }
                }
                uint8_t* dst = sQ + (u >> 1) * kQBlk;
#pragma unroll
                for (int c = 0; c < 4; c++) {
                    uint4 w;
                    w.x = pack_bf16x2(v[8 * c], v[8 * c + 1]);
                    w.y = pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
                    w.z = pack_bf16x2(v[8 * c + 4], v[8 * c + 5]);
                    w.w = pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
                    *reinterpret_cast<uint4*>(dst + swz(hq, (u & 1) * 4 + c)) = w;
                }
            }
            if (x.tile0 == 0) {
                // window row r = i / 2; thread u = i % 2 takes channels u*32 .. u*32+31 and
                // 64 + u*32 .. 64 + u*32+31 (16 RoPE pairs each): RMSNorm over the row (the
                // pair's sums of squares added), RoPE at the row's position, bf16, swizzled
                const int r = i >> 1, u = i & 1;
                const int64_t p = (int64_t)x.w0 + r;
                bool valid = r < x.n_win;
                if (valid && p < a.raw.first(x.b, a.seq_len[x.b])) {
                    valid = false;
                    flag(a.st, CSA_DEV_OOB);
                }
                float v[64];
                float ss = 0.f;
                if (valid) {
                    const uint16_t* src = a.kv + a.raw.row(x.b, p) * kD + u * 32;
#pragma unroll
                    for (int c = 0; c < 8; c++) {
                        const uint4 w = *reinterpret_cast<const uint4*>(src + (c >> 2) * 64 + 8 * (c & 3));
                        const uint32_t w4[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
                        for (int z = 0; z < 4; z++) {
                            const float2 f = bf16x2_to_f32(w4[z]);
                            v[8 * c + 2 * z] = f.x;
                            v[8 * c + 2 * z + 1] = f.y;
                            ss += f.x * f.x + f.y * f.y;
                        }
                    }
                } else {
#pragma unroll
                    for (int c = 0; c < 64; c++) v[c] = 0.f;
                }
                ss += __shfl_xor_sync(0xffffffffu, ss, 1);
                if (valid) {
                    const float rn = rsqrtf(ss / (float)kD + a.eps);
#pragma unroll
                    for (int c = 0; c < 64; c++) v[c] *= rn;
                    // angle (w0 + r) f_j = w0 f_j + r f_j: the first term from the fp64 table,
                    // the second (< 128 rad) by sincosf; combined by the addition formula
#pragma unroll
                    for (int k = 0; k < 16; k++) {
                        const int pj = u * 16 + k;
                        float sb, cb;
                        sincosf((float)r * rf[pj], &sb, &cb);
                        const float cs = rwc[pj] * cb - rws[pj] * sb, sn = rws[pj] * cb + rwc[pj] * sb;
                        const float x0 = v[32 + 2 * k], y0 = v[32 + 2 * k + 1];
                        v[32 + 2 * k] = x0 * cs - y0 * sn;
                        v[32 + 2 * k + 1] = x0 * sn + y0 * cs;
                    }
                }
#pragma unroll
                for (int c = 0; c < 8; c++) {
                    uint4 w;
                    w.x = pack_bf16x2(v[8 * c], v[8 * c + 1]);
                    w.y = pack_bf16x2(v[8 * c + 2], v[8 * c + 3]);
                    w.z = pack_bf16x2(v[8 * c + 4], v[8 * c + 5]);
                    w.w = pack_bf16x2(v[8 * c + 6], v[8 * c + 7]);
                    *reinterpret_cast<uint4*>(sW + (c >> 2) * kBlk + swz(r, u * 4 + (c & 3))) = w;
                }
            }
            fence_async_smem();
            // all warps' stores (including the window mask) before anyone reads them
            asm volatile("bar.sync 1, 256;" ::: "memory");
            __syncwarp();
            if (lane == 0) mbar_arrive(prep_full);

            // sparse: the sink of head h0 + i of this rank's slice, for the combine
            float sk_mine = -INFINITY;
            if (a.idx) {
                const int h0 = x.c * kH / a.cluster, h1 = (x.c + 1) * kH / a.cluster;
                if (i < h1 - h0) sk_mine = h0 + i < a.hreal ? a.sink[h0 + i] * kLog2e : -INFINITY;
            }
            // ---- running state of (head h, column-half ch) ----
            // the chunk's own keys only: the sink enters when the partial states are combined.
            // mref is the reference maximum of P = 2^(s - mref); it moves only when a tile's
            // maximum exceeds it by more than 2^kRescale, and then O_ch is rescaled in TMEM.
            float mref = -INFINITY;
            float lrun = 0.f;
            for (int jj = 0; jj < x.ntiles && ok; jj++) {
                const int j = x.tile0 + jj;
                const int sb = nt & 1;
                if (!mbar_wait_warp(&s_full[sb], (nt >> 1) & 1, abort_flag, a.st)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                uint32_t sv[32];
                tmem_ld32(tmem_S + sb * 64 + ch * 32 + lane_base, sv);
                tmem_ld_wait();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&s_empty[sb]);
                // validity of my 32 keys (the MMA has consumed the tile, so its mask is stable
                // until the producer refills the stage after this tile's P.V)
                const uint32_t* mk = smask + (j == 0 ? kStages : kst) * 4;
                if (j != 0 && ++kst == kStages) kst = 0;
                const uint32_t mw = mk[2 * kh + ch];
                // raw scores (masked keys -inf); the scale is positive, so the maximum of the
                // scaled scores is the scaled maximum
                float rmax = -INFINITY;
                if (mw == 0xffffffffu) {
#pragma unroll
                    for (int c = 0; c < 32; c++) rmax = fmaxf(rmax, __uint_as_float(sv[c]));
                } else {
#pragma unroll
                    for (int c = 0; c < 32; c++) {
                        const float xv = ((mw >> c) & 1u) ? __uint_as_float(sv[c]) : -INFINITY;
                        sv[c] = __float_as_uint(xv);
                        rmax = fmaxf(rmax, xv);
                    }
                }
                float tmax = rmax * a.scale_log2;
                tmax = fmaxf(tmax, __shfl_xor_sync(0xffffffffu, tmax, 16));
                const bool need = tmax > mref + kRescale;
                if (__any_sync(0xffffffffu, need)) {
                    const float mnew = need ? tmax : mref;
                    const float corr = !need ? 1.f : (mref == -INFINITY ? 0.f : exp2f(mref - mnew));
                    if (jj > 0 && __any_sync(0xffffffffu, corr != 1.f)) {
                        // O_ch must hold every earlier P V of the item before it is rescaled.
                        // P V of tile nt - 2 is complete once this tile's P buffer is free;
                        // then pvdone has completed nt - 1 or nt phases, and its parity wait
                        // for phase nt - 1 cannot alias an older one
                        if (!mbar_wait_warp(&p_empty[sb], ((nt >> 1) & 1) ^ 1, abort_flag, a.st) ||
                            !mbar_wait_warp(pvdone, (nt - 1) & 1, abort_flag, a.st)) {
                            ok = false;
                            break;
                        }
                        tc_fence_after();
#pragma unroll 1
                        for (int cc = 0; cc < 4; cc++) {
                            uint32_t ov[16];
                            const uint32_t col = tmem_O + ch * 64 + 16 * cc + lane_base;
                            tmem_ld16(col, ov);
                            tmem_ld_wait();
#pragma unroll
                            for (int z = 0; z < 16; z++)
                                ov[z] = __float_as_uint(__uint_as_float(ov[z]) * corr);
                            tmem_st16(col, ov);
                        }
                        tmem_st_wait();
                        tc_fence_before();
                    }
                    lrun *= corr;
                    mref = mnew;
                }
                // P = 2^(s * scale - mref): one FMA and one ex2 per key (a masked key is -inf,
                // giving 0); with no valid key yet (mref = -inf) every P of the tile is 0
                float rs = 0.f;
                uint32_t pk[16];
                if (mref == -INFINITY) {
#pragma unroll
                    for (int c = 0; c < 16; c++) pk[c] = 0u;
                } else {
                    const float nm = -mref;
#pragma unroll
                    for (int c = 0; c < 16; c++) {
                        const float p0 = ex2_approx(fmaf(__uint_as_float(sv[2 * c]), a.scale_log2, nm));
                        const float p1 = ex2_approx(fmaf(__uint_as_float(sv[2 * c + 1]), a.scale_log2, nm));
                        rs += p0 + p1;
                        pk[c] = pack_bf16x2(p0, p1);
                    }
                }
                rs += __shfl_xor_sync(0xffffffffu, rs, 16);
                lrun += rs;
                // P (bf16) into shared memory: head h, keys kh*64 + ch*32 .. +31
                if (!mbar_wait_warp(&p_empty[sb], ((nt >> 1) & 1) ^ 1, abort_flag, a.st)) {
                    ok = false;
                    break;
                }
                uint8_t* prow = sP + sb * 2 * kPBlk + kh * kPBlk;
#pragma unroll
                for (int c = 0; c < 4; c++)
                    *reinterpret_cast<uint4*>(prow + swz(h, ch * 4 + c)) =
                        make_uint4(pk[4 * c], pk[4 * c + 1], pk[4 * c + 2], pk[4 * c + 3]);
                fence_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(&p_full[sb]);
                nt++;
            }
            // ---- the item's output: O_ch from TMEM, the two column-halves merged ----
            if (ok) ok = mbar_wait_warp(odone, nitem & 1, abort_flag, a.st);
            // the stores below (out, or the chunk partials of the workspace) may overwrite
            // what the previous kernel still reads (an earlier call's combine on the same
            // workspace); a window-only item reaches them without passing the producer's
            // wait, so every thread here waits for the previous grid once
            if (!waited_prev) {
                pdl_wait();
                waited_prev = true;
            }
            float o[64];
            {
                uint32_t ov[64];
#pragma unroll
                for (int c = 0; c < 64; c++) ov[c] = 0u;
                if (ok) {
                    tc_fence_after();
                    tmem_ld64(tmem_O + ch * 64 + lane_base, ov);
                    tmem_ld_wait();
                    tc_fence_before();
                }
#pragma unroll
                for (int c = 0; c < 64; c++) o[c] = __uint_as_float(ov[c]);
            }
            // column-half 1 hands its state to column-half 0 through the idle window buffer
            // (every MMA of the item is complete), thread slot = quarter * 32 + lane
            float* xo = reinterpret_cast<float*>(sW);
            const int slot = quarter * 32 + lane;
            if (ok && ch == 1) {
#pragma unroll
                for (int c = 0; c < 64; c++) xo[c * 128 + slot] = o[c];
                xml[2 * slot] = mref;
                xml[2 * slot + 1] = lrun;
            }
            if (!named_barrier_and(1, 256, ok)) {
                ok = false;
                break;
            }
            float mrun = mref;
            if (ch == 0) {
                const float m1 = xml[2 * slot], l1 = xml[2 * slot + 1];
                mrun = fmaxf(mref, m1);
                const float w0 = mref == -INFINITY ? 0.f : exp2f(mref - mrun);
                const float w1 = m1 == -INFINITY ? 0.f : exp2f(m1 - mrun);
                lrun = lrun * w0 + l1 * w1;
#pragma unroll
                for (int c = 0; c < 64; c++) o[c] = o[c] * w0 + xo[c * 128 + slot] * w1;
            }
            if (a.idx) {
                // ---- sparse: exchange partial states across the cluster ----
                const int C = a.cluster;
                const int nh = (kH + C - 1) / C;
                float* recv_ml = recv + C * nh * kD;
                if (ch == 0) {
                    // every rank's receive buffer is free of the previous query's partials
                    ok = mbar_wait_cluster_warp(cpart_free, (nitem & 1) ^ 1, abort_flag, a.st);
                    if (ok) {
                        // head h is finished by rank `own` (heads [own*kH/C, (own+1)*kH/C))
                        int own = 0;
                        while (own + 1 < C && (own + 1) * kH / C <= h) own++;
                        const int lh = h - own * kH / C;
                        const uint32_t dst = mapa(recv + ((x.c * nh + lh) * kD + kh * 64), (uint32_t)own);
#pragma unroll
                        for (int c = 0; c < 64; c += 4)
                            st_cluster_f4(dst + 4 * c, make_float4(o[c], o[c + 1], o[c + 2], o[c + 3]));
                        if (kh == 0) {
                            st_cluster_f32(mapa(recv_ml + (2 * x.c) * nh + lh, (uint32_t)own), mrun);
                            st_cluster_f32(mapa(recv_ml + (2 * x.c + 1) * nh + lh, (uint32_t)own), lrun);
                        }
                        fence_cluster();
                        __syncwarp();
                        if (lane == 0)
                            for (int r = 0; r < C; r++) mbar_arrive_cluster(mapa(cpart_full, (uint32_t)r));
                        ok = mbar_wait_cluster_warp(cpart_full, nitem & 1, abort_flag, a.st);
                    }
                }
                if (named_barrier_and(1, 256, ok)) {
                    // this rank's heads; first the combine weights, one thread per head:
                    // M = max(sink, m_r), w_r = 2^(m_r - M), L = 2^(sink - M) + sum_r w_r l_r
                    const int h0 = x.c * kH / C, h1 = (x.c + 1) * kH / C;
                    if (i < h1 - h0) {
                        const float sk = sk_mine;
                        float M = sk;
                        for (int r = 0; r < C; r++) M = fmaxf(M, recv_ml[(2 * r) * nh + i]);
                        float L = (M == -INFINITY || sk == -INFINITY) ? 0.f : exp2f(sk - M);
                        for (int r = 0; r < C; r++) {
                            const float mr = recv_ml[(2 * r) * nh + i];
                            const float w = (mr == -INFINITY) ? 0.f : exp2f(mr - M);
                            L = fmaf(w, recv_ml[(2 * r + 1) * nh + i], L);
                            wtab[i * (kMaxCluster + 1) + r] = w;
                        }
                        wtab[i * (kMaxCluster + 1) + kMaxCluster] = L;
                    }
                    asm volatile("bar.sync 1, 256;" ::: "memory");
                    // then (head, 4 channels) per work unit: sum_r w_r O_r / L, inverse RoPE
                    // (the pairs sit inside the 4 channels), 4 bf16 stored at once
                    const int units = (h1 - h0) * (kD / 4);
#pragma unroll 2
                    for (int w = i; w < units; w += 256) {
                        const int lh = w / (kD / 4), c4 = (w % (kD / 4)) * 4;
                        const float* wt = wtab + lh * (kMaxCluster + 1);
                        float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
                        for (int r = 0; r < C; r++) {
                            const float wr = wt[r];
                            const float4 v = *reinterpret_cast<const float4*>(recv + (r * nh + lh) * kD + c4);
                            acc.x = fmaf(wr, v.x, acc.x);
                            acc.y = fmaf(wr, v.y, acc.y);
                            acc.z = fmaf(wr, v.z, acc.z);
                            acc.w = fmaf(wr, v.w, acc.w);
                        }
                        const float L = wt[kMaxCluster];
                        if (L > 0.f) {
                            acc.x /= L;
                            acc.y /= L;
                            acc.z /= L;
                            acc.w /= L;
                        } else {
                            acc = make_float4(0.f, 0.f, 0.f, 0.f);
                        }
                        if (c4 >= kD - kRopeDims) {
                            // rotation by -t: (x, y) -> (x cos + y sin, y cos - x sin)
                            const int pj = (c4 - (kD - kRopeDims)) >> 1;
                            const float c0 = rqc[pj], s0 = rqs[pj], c1 = rqc[pj + 1], s1 = rqs[pj + 1];
                            acc = make_float4(acc.x * c0 + acc.y * s0, acc.y * c0 - acc.x * s0,
                                              acc.z * c1 + acc.w * s1, acc.w * c1 - acc.z * s1);
                        }
                        if (h0 + lh < a.hreal)
                            *reinterpret_cast<uint2*>(a.out + ((int64_t)x.q * a.hreal + h0 + lh) * kD + c4) =
                                make_uint2(pack_bf16x2(acc.x, acc.y), pack_bf16x2(acc.z, acc.w));
                    }
                    // every thread's reads of the receive buffer are done; then it may take
                    // the next query's partials
                    asm volatile("bar.sync 1, 256;" ::: "memory");
                    if (ch == 0) {
                        fence_cluster();
                        __syncwarp();
                        if (lane == 0)
                            for (int r = 0; r < C; r++) mbar_arrive_cluster(mapa(cpart_free, (uint32_t)r));
                    }
                } else {
                    ok = false;
                }
            } else if (ok && ch == 0) {
                float* pr = a.part + ((int64_t)it * kH + h) * (kD + 2);
                if (kh == 0) {
                    pr[0] = mrun;
                    pr[1] = lrun;
                }
                // rows are kD + 2 floats: 8-byte aligned
#pragma unroll
                for (int c = 0; c < 64; c += 2)
                    *reinterpret_cast<float2*>(pr + 2 + kh * 64 + c) = make_float2(o[c], o[c + 1]);
            }
            nitem++;
            if (ok) combine_here(it);
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, 256);
    }
    // no rank leaves while another may still read its shared memory or arrive on it
    if (a.cluster > 1) cluster_sync_all();
}

// Dense path, spread variant: combine the chunk partials of one (query, head) (see
// combine_pair).  Thread = pair of channels.
__global__ void __launch_bounds__(kD / 2) attn_combine_kernel(const AttnTcArgs a) {
    const int q = blockIdx.y, h = blockIdx.x, d = 2 * threadIdx.x;
    // query metadata is an input: read before the wait on the attention kernel
    int t;
    const int nch = dense_chunks(a, q, t);
    pdl_wait();   // chunk partials come from the attention kernel
    pdl_trigger();
    if (nch == 0 || h >= a.hreal) return;
    const float2 o = combine_pair(a, q, t, nch, h, d);
    *reinterpret_cast<uint32_t*>(a.out + ((int64_t)q * a.hreal + h) * kD + d) = pack_bf16x2(o.x, o.y);
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult qr;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &qr) ==
                cudaSuccess &&
            qr == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    });
    return fn;
}

int sm_count() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

constexpr size_t kSmemBytes = 1024 + kStages * kTileBytes + kTileBytes + 2 * kQBlk + 4 * kPBlk +
                              4 * (kStages + 1) * 4 + 5 * 32 * 4 + kMaxK * 4 + kStages * kTK * 4 +
                              (kRecvFloats + kWtabFloats + 256) * 4 + (2 * kStages + 17) * 8 + 16;
static_assert(kSmemBytes <= 232448, "shared memory per CTA");
static_assert((kRecvFloats + kWtabFloats + 256) % 2 == 0, "mbarriers 8-byte aligned");

// CTAs per query for sparse attention, a function of k alone (so the result is
// batch-invariant).  Up to 4 selected-entry tiles (k <= 512, decode): a cluster whose rank
// 0 takes the window tile and the others about two entry tiles each, for latency.  More
// (k >= 1024, as in prefill chunks of thousands of queries): one CTA per query over every
// tile, persistent over queries, which saves each query's cross-CTA exchange.
int sparse_cluster(int k) {
    const int n_et = (k + kTK - 1) / kTK;
    if (n_et >= 8) return 1;
    return min(kMaxCluster, 1 + (n_et + 1) / 2);
}

// Clusters of `C` CTAs that can be resident at once (0 when unknown).
int max_active_clusters(int C) {
    static int cache[kMaxCluster + 1] = {};
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    if (cache[C] == 0) {
        cudaLaunchConfig_t cfg = {};
        cfg.gridDim = dim3(C * 64);
        cfg.blockDim = dim3(kThreads);
        cfg.dynamicSmemBytes = kSmemBytes;
        cudaLaunchAttribute attr[1];
        attr[0].id = cudaLaunchAttributeClusterDimension;
        attr[0].val.clusterDim.x = (unsigned)C;
        attr[0].val.clusterDim.y = 1;
        attr[0].val.clusterDim.z = 1;
        cfg.attrs = attr;
        cfg.numAttrs = 1;
        int n = 0;
        if (cudaOccupancyMaxActiveClusters(&n, attn_tc_kernel, &cfg) != cudaSuccess || n <= 0) {
            cudaGetLastError();
            n = sm_count() / C;
        }
        cache[C] = n;
    }
    return cache[C];
}

// the window chunk, then the entry tiles in chunks of kDenseChunkTiles
int dense_chunks_per_q(int max_n) {
    return 1 + ((max_n + kTK - 1) / kTK + kDenseChunkTiles - 1) / kDenseChunkTiles;
}

}  // namespace

// 16-head calls run on the 64-head tile, the other heads zero (their outputs are not stored)
bool attn_tc_supported(int H, int D, int fmt) {
    return (H == kH || H == 16) && D == kD && fmt == CSA_KV_BF16;
}

size_t attn_tc_workspace_bytes(int Q, int max_n) {
    return (size_t)Q * dense_chunks_per_q(max_n) * kH * (kD + 2) * sizeof(float);
}

cudaError_t launch_attn_tc(const AttnArgs& aa, int Q, int max_n, void* workspace,
                           cudaStream_t stream) {
    if (Q == 0) return cudaSuccess;
    AttnTcArgs a;
    a.q = aa.q;
    a.entries = aa.entries;
    a.er = aa.er;
    a.kv = aa.kv;
    a.raw = aa.raw;
    a.q_seq = aa.q_seq;
    a.q_pos = aa.q_pos;
    a.seq_len = aa.seq_len;
    a.idx = aa.idx;
    a.sink = aa.sink;
    a.out = aa.out;
    a.part = reinterpret_cast<float*>(workspace);
    a.st = aa.st;
    a.ent_rows = aa.ent_rows;
    a.k = aa.k;
    a.m = aa.m;
    a.B = aa.B;
    a.W = aa.W;
    a.Q = Q;
    a.max_n = max_n;
    a.scale_log2 = aa.scale * kLog2e;
    a.eps = aa.eps;
    a.log2_theta = aa.log2_theta;
    a.hreal = aa.H;
    if (aa.idx) {
        a.cluster = sparse_cluster(aa.k);
        a.chunk_tiles = 0;   // ranks take their tiles by rank
        a.chunks_per_q = a.cluster;
    } else {
        a.cluster = 1;
        a.chunk_tiles = kDenseChunkTiles;
        a.chunks_per_q = dense_chunks_per_q(max_n);
    }
    // dense: the query's chunks spread over CTAs (low latency while the chunks of the batch
    // leave SMs idle otherwise), or one CTA per query from as many queries as SMs on (high
    // throughput: no combine kernel, each query's partials stay with its CTA).  Both give the
    // same bits, so the choice may follow the batch.
    a.single = (!aa.idx && Q >= sm_count()) ? 1 : 0;
    a.total_items = Q * a.chunks_per_q;
    // dense: 128-row boxes of contiguous entries; sparse: one-row boxes for 4-row gathers
    CUtensorMap map_e, map_g;
    std::memset(&map_e, 0, sizeof(map_e));
    std::memset(&map_g, 0, sizeof(map_g));
    if (aa.ent_rows > 0) {
        EncodeFn enc = encode_fn();
        if (!enc) return cudaErrorInvalidValue;
        const cuuint64_t dims[2] = {(cuuint64_t)kD, (cuuint64_t)aa.ent_rows};
        const cuuint64_t strides[1] = {(cuuint64_t)kD * 2};
        const cuuint32_t box[2] = {64, aa.idx ? 1u : (cuuint32_t)kTK};
        const cuuint32_t estr[2] = {1, 1};
        if (enc(aa.idx ? &map_g : &map_e, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
                const_cast<uint8_t*>(aa.entries), dims, strides, box, estr,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return cudaErrorInvalidValue;
    }
    cudaError_t e = cudaFuncSetAttribute(attn_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)kSmemBytes);
    if (e != cudaSuccess) return e;
    {
        LaunchScope scope(kKAttnTc, stream);
        if (aa.idx) {
            // one cluster per query at a time; clusters walk the queries persistently
            const int nclusters = max(1, min(Q, max_active_clusters(a.cluster)));
            e = launch_pdl_cluster(attn_tc_kernel, dim3(nclusters * a.cluster), dim3(kThreads),
                                   kSmemBytes, stream, a.cluster, map_e, map_g, a);
        } else {
            const int grid = min(a.single ? Q : a.total_items, sm_count());
            e = launch_pdl(attn_tc_kernel, dim3(grid), dim3(kThreads), kSmemBytes, stream, map_e,
                           map_g, a);
        }
    }
    if (e != cudaSuccess || aa.idx || a.single) return e;
    LaunchScope scope(kKAttnCombine, stream);
    return launch_pdl(attn_combine_kernel, dim3(kH, Q), dim3(kD / 2), 0, stream, a);
}

}  // namespace csa
