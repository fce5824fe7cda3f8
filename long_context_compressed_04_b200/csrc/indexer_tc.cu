// Step a3 on the 5th-generation tensor cores: lightning-indexer scores.
//
// "DeepSeek-V4 深度分析报告" 2.1 CSA: the lightning indexer scores every visible
// compressed entry for the query; s_i = ks_i * sum_h (w_h * qs_h) * ReLU(q_h . k_i), the
// heads accumulated by fmaf in ascending order in fp32 (the definition all paths share).
//
// Decode is HBM-bound (each 132-byte key row is read once and feeds 64 x 128 MACs, about
// 124 FLOP/byte), but that intensity still needs the tensor pipe to keep up with HBM.
// Work is counted in tiles of 128 entries, aligned to each query's sequence; query q owns
// the tiles [q * T, q * T + T) of a virtual tile space (T = tiles of the longest query).
// One persistent CTA per SM takes an equal contiguous range of that space and walks it as
// items: the pieces of the range cut at query boundaries and every 8 tiles.  Every entry
// is always computed in the same tile row by the same instructions whatever the batch.
// Roles per CTA (11 warps):
//   warp 0 lane 0  TMA producer: per query the heads (H_I x d_I e4m3, B operand, reused
//                  across consecutive items of the query); per stage a group of up to four
//                  tiles of 128 key rows (A operand), 128-byte swizzle for d_I = 128 and
//                  64-byte swizzle for d_I = 64, a 3-stage ring; it decodes its items itself
//                  and starts before the others' item table;
//   warp 1         TMEM allocation; lane 0 issues tcgen05.mma kind::f8f6f4 (M=128 entries,
//                  N=H_I heads, d_I / 32 x K=32 per tile) into one of two sets of four TMEM
//                  accumulators, the K steps of the group's tiles interleaved;
//   warp 2         item prefetch: w_h * qs_h of the item's query and the key scales of
//                  its tiles into a shared-memory ring, ahead of the epilogue;
//   warps 3-10     epilogue in two groups of four taking alternate tiles of a group:
//                  tcgen05.ld of one entry row (all heads) per thread, the fixed-order fmaf
//                  chain, the key scale, a coalesced score store.
// Head counts below 16, 32 or 64 run on the next of those MMA widths: the padded heads'
// rows of the B operand are zero and their weights w_h * qs_h are zero, so each adds an
// exact +0 to the fmaf chain and the scores keep their bits.
// Barriers are per group of tiles, not per tile: under load every mbarrier operation costs
// the single issuing thread on the order of a hundred cycles.
// Every wait is bounded; a timeout aborts the CTA, drains its own copies and MMAs,
// frees TMEM and reports CSA_DEV_TIMEOUT.
#include <mutex>

#include "launchers.cuh"
#include "indexer_items.cuh"
#include "sm100.cuh"

namespace csa {

namespace {

constexpr int kGroupTiles = 4;           // tiles per pipeline stage (one barrier each way)
constexpr int kStages = 3;               // 3 x 64 KB of key tiles in flight per SM
constexpr int kAccSets = 2;              // TMEM accumulator sets of kGroupTiles accumulators
constexpr int kAux = 3;                  // prefetched items
constexpr int kFirstEpiWarp = 3;
constexpr int kEpiWarps = 8;
constexpr int kThreads = 32 * (kFirstEpiWarp + kEpiWarps);

struct IdxArgs {
    const float* qs;
    const float* w;
    const float* ks;
    const int64_t* seq_len;
    EntryRows er;            // where entry i of sequence b lies (contiguous or block table)
    const int32_t* q_seq;
    const int32_t* q_pos;
    float* scores;
    int64_t ld;
    int64_t ent_rows;
    int32_t* st;
    int Q, B, m, max_n;
    int hreal;               // heads of the call (<= HI; the rest are zero padding)
    int keys_once;           // no more queries than sequences (decode): each key row is read once
    int qtiles;              // virtual tiles per query: ceil(max_n / 128)
    int chunks_per_q;        // ceil(qtiles / 8)
    // nullable: per query, the largest score key (order_key) of every group of 32
    // consecutive entries, group g of query q at gmax[q * ld_g + g] (see the top-k)
    uint32_t* gmax;
    int64_t ld_g;
};

// TMEM columns: kAccSets x kGroupTiles accumulators of HI fp32 columns, rounded to a power
// of two >= 32.
template <int HI>
__host__ __device__ constexpr uint32_t tmem_cols() {
    constexpr int c = kAccSets * kGroupTiles * HI;
    return c <= 32 ? 32u : c <= 64 ? 64u : c <= 128 ? 128u : c <= 256 ? 256u : 512u;
}

// Floats of one prefetch slot: w*qs for the heads, then the key scales of up to 8 tiles.
template <int HI>
__host__ __device__ constexpr int aux_floats() {
    return HI + kChunkTiles * kTileRows;
}

// Bytes of one tile of 128 key rows of DI e4m3.
template <int DI>
__host__ __device__ constexpr int tile_bytes() {
    return kTileRows * DI;
}

// HI: MMA width (heads, padded); DI: indexer dim (MMA K total, bytes per key row).
// PAGED: the key rows come through the block table (a separate instantiation, so the
// contiguous kernel carries no block-table code).
template <int HI, int DI, bool PAGED>
__global__ void __launch_bounds__(kThreads, 1)
    indexer_tc_kernel(const __grid_constant__ CUtensorMap tmap_k,
                      const __grid_constant__ CUtensorMap tmap_q, const IdxArgs a) {
    using namespace sm100;
    static_assert(DI == 64 || DI == 128, "indexer dim 64 or 128");
    constexpr int kTileBytes = tile_bytes<DI>();
    constexpr int kGroupBytes = kGroupTiles * kTileBytes;
    constexpr int kQBytes = HI * DI;
    constexpr int kAuxFloats = aux_floats<HI>();
    constexpr uint32_t kIdesc = instr_desc(0, 0, kTileRows, HI);
    extern __shared__ __align__(1024) uint8_t smem_raw[];
    uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                               ~uintptr_t(1023));
    uint8_t* sA = smem;                                  // [kStages][kGroupTiles][128 x DI]
    uint8_t* sB = sA + kStages * kGroupBytes;            // [2][HI x DI]
    float* aux = reinterpret_cast<float*>(sB + 2 * kQBytes);   // [kAux][kAuxFloats]
    uint64_t* bars = reinterpret_cast<uint64_t*>(aux + kAux * kAuxFloats);
    uint64_t* full = bars;                               // [kStages]
    uint64_t* empty = full + kStages;                    // [kStages]
    uint64_t* bfull = empty + kStages;                   // [2]
    uint64_t* bempty = bfull + 2;                        // [2]
    uint64_t* accfull = bempty + 2;                      // [kAccSets]
    uint64_t* accempty = accfull + kAccSets;             // [kAccSets]
    uint64_t* auxfull = accempty + kAccSets;             // [kAux]
    uint64_t* auxempty = auxfull + kAux;                 // [kAux]
    uint64_t* drain = auxempty + kAux;                   // [1]
    uint32_t* tmem_base_smem = reinterpret_cast<uint32_t*>(drain + 1);
    volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_base_smem + 1);
    Item* items = reinterpret_cast<Item*>(tmem_base_smem + 4);   // [kMaxItems]
    int64_t v0, v1;
    cta_range(a, blockIdx.x, gridDim.x, v0, v1);
    const int n_my = v1 > v0 ? (int)(chunk_of(a, v1 - 1) - chunk_of(a, v0) + 1) : 0;

    // The indexer reads only its inputs (keys, query heads, weights and scales), never an
    // earlier libcsa kernel's output, so its loads and MMAs may overlap the kernel before
    // it.  Its score stores may not: an earlier top-k can still be reading the same score
    // rows (two calls in a row on one workspace), so every epilogue thread waits for the
    // previous grid before its first store.  The next kernel (the top-k, which waits for
    // this grid before reading) may launch right away; the wait at the end keeps
    // completion ordered for the kernels after it.
    pdl_trigger();
    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    if (threadIdx.x == 0) {
        for (int s = 0; s < kStages; s++) {
            mbar_init(&full[s], 1);
            mbar_init(&empty[s], 1);
        }
        for (int i = 0; i < 2; i++) {
            mbar_init(&bfull[i], 1);
            mbar_init(&bempty[i], 1);
        }
        for (int i = 0; i < kAccSets; i++) {
            mbar_init(&accfull[i], 1);
            mbar_init(&accempty[i], kEpiWarps);
        }
        for (int i = 0; i < kAux; i++) {
            mbar_init(&auxfull[i], 32);               // every lane of the prefetch warp
            mbar_init(&auxempty[i], kEpiWarps);
        }
        mbar_init(drain, 1);
        *abort_flag = 0;
        mbar_fence_init();
        prefetch_tmap(&tmap_k);
        prefetch_tmap(&tmap_q);
    }
    if (warp == 1) {
        tmem_alloc(tmem_base_smem, tmem_cols<HI>());
        tmem_relinquish();
    }
    if (a.hreal < HI) {
        // the padded heads' B rows stay zero: the copies write rows [0, hreal) only.  The
        // swizzle permutes 16-byte pieces within a row, so rows [hreal, HI) are exactly the
        // bytes from hreal * DI on in each buffer.
        for (int u = threadIdx.x; u < 2 * (HI - a.hreal) * DI / 16; u += kThreads) {
            const int per = (HI - a.hreal) * DI / 16;
            const int bb = u / per, o = u % per;
            reinterpret_cast<uint4*>(sB + bb * kQBytes + a.hreal * DI)[o] = make_uint4(0u, 0u, 0u, 0u);
        }
        fence_proxy_async_smem();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem_base = *tmem_base_smem;
    if (warp > 0) {
        // every role but the producer resolves the items' metadata (dependent loads) in
        // parallel, once; items past the table are decoded on the fly
        for (int i = threadIdx.x - 32; i < min(n_my, kMaxItems); i += kThreads - 32) {
            Item x;
            if (!get_item(a, v0, v1, i, x, true)) x.ntiles = 0;
            items[i] = x;
        }
        asm volatile("bar.sync 1, %0;" ::"r"(kThreads - 32) : "memory");
    }

    if (warp == 0) {
        if (lane == 0) {
            // ---------------- TMA producer ----------------
            int stage = 0;
            uint32_t ephase = 0;
            int nq = 0, cur_q = -1, ng = 0;   // queries and groups issued
            bool ok = true;
            // key rows read once (decode) take the evict-first policy: the key tiles
            // leave L2 first, and the score rows and group maxima the top-k reads next stay
            const uint64_t pol = l2_policy(a.keys_once != 0);
            for (int ii = 0; ii < n_my && ok; ii++) {
                Item x;
                if (!get_item(a, v0, v1, ii, x, false)) continue;
                if (x.q != cur_q) {
                    const int bb = nq & 1;
                    if (!mbar_wait(&bempty[bb], ((nq >> 1) & 1) ^ 1, abort_flag, a.st)) break;
                    mbar_arrive_expect_tx(&bfull[bb], (uint32_t)(a.hreal * DI));
                    tma_load_2d(sB + bb * kQBytes, &tmap_q, &bfull[bb], 0, x.q * a.hreal);
                    nq++;
                    cur_q = x.q;
                }
                for (int g0 = 0; g0 < x.ntiles; g0 += kGroupTiles) {
                    const int gt = min(kGroupTiles, x.ntiles - g0);
                    if (!mbar_wait(&empty[stage], ephase ^ 1, abort_flag, a.st)) {
                        ok = false;
                        break;
                    }
                    if constexpr (!PAGED) {
                        mbar_arrive_expect_tx(&full[stage], gt * kTileBytes);
                        for (int j = 0; j < gt; j++)
                            tma_load_2d_hint(sA + stage * kGroupBytes + j * kTileBytes, &tmap_k, &full[stage], 0,
                                             (int32_t)(x.row0 + (int64_t)(x.tile0 + g0 + j) * kTileRows), pol);
                    } else {
                        // block table: each tile in blocks of kPageRows rows (the map's box)
                        int32_t rows[kGroupTiles][kTilePages];
                        int nb = 0;
                        for (int j = 0; j < gt; j++) nb += tile_pages(a, x, x.tile0 + g0 + j, rows[j]);
                        mbar_arrive_expect_tx(&full[stage], (uint32_t)nb * (kPageRows * DI));
                        for (int j = 0; j < gt; j++)
#pragma unroll
                            for (int p = 0; p < kTilePages; p++)
                                if (rows[j][p] >= 0)
                                    tma_load_2d_hint(sA + stage * kGroupBytes + j * kTileBytes + p * (kPageRows * DI),
                                                     &tmap_k, &full[stage], 0, rows[j][p], pol);
                    }
                    ng++;
                    if (++stage == kStages) {
                        stage = 0;
                        ephase ^= 1;
                    }
                }
            }
            // drain: every copy this thread issued must have landed before smem is released
            for (int s = 0; s < kStages; s++) {
                const int cnt = ng / kStages + (s < ng % kStages ? 1 : 0);
                if (cnt) mbar_drain(&full[s], (cnt - 1) & 1, a.st);
            }
            for (int i = 0; i < 2; i++) {
                const int cnt = (nq - i + 1) / 2;
                if (cnt) mbar_drain(&bfull[i], (cnt - 1) & 1, a.st);
            }
        }
    } else if (warp == 1) {
        if (lane == 0) {
            // ---------------- MMA issuer ----------------
            // One stage = one group of up to four tiles of one item.  The K steps of the
            // group's tiles are interleaved across their accumulators: a small-N MMA chained
            // on one accumulator waits for the previous one, so independent chains keep the
            // tensor pipe busy.
            int stage = 0;
            uint32_t sphase = 0;
            int nq = 0, cur_q = -1, ng = 0;
            uint64_t bdesc = 0;
            bool ok = true;
            for (int ii = 0; ii < n_my && ok; ii++) {
                Item x;
                if (!fetch_item(a, items, v0, v1, ii, x, false)) continue;
                if (x.q != cur_q) {
                    // the previous query's heads are free once the MMAs issued so far finish
                    if (nq > 0) mma_commit(&bempty[(nq - 1) & 1]);
                    const int bb = nq & 1;
                    if (!mbar_wait(&bfull[bb], (nq >> 1) & 1, abort_flag, a.st)) break;
                    tc_fence_after();
                    if constexpr (DI == 128)
                        bdesc = smem_desc_k_sw128(sB + bb * kQBytes);
                    else
                        bdesc = smem_desc_k_sw64(sB + bb * kQBytes);
                    nq++;
                    cur_q = x.q;
                }
                for (int g0 = 0; g0 < x.ntiles; g0 += kGroupTiles) {
                    const int gt = min(kGroupTiles, x.ntiles - g0);
                    const int set = ng & (kAccSets - 1);
                    if (!mbar_wait(&accempty[set], ((ng / kAccSets) & 1) ^ 1, abort_flag, a.st) ||
                        !mbar_wait(&full[stage], sphase, abort_flag, a.st)) {
                        ok = false;
                        break;
                    }
                    tc_fence_after();
                    const uint64_t adesc = DI == 128 ? smem_desc_k_sw128(sA + stage * kGroupBytes)
                                                     : smem_desc_k_sw64(sA + stage * kGroupBytes);
                    const uint32_t d0 = tmem_base + (uint32_t)(set * kGroupTiles * HI);
#pragma unroll
                    for (int kk = 0; kk < DI / 32; kk++) {   // K = 32 e4m3 = 32 bytes per MMA
#pragma unroll
                        for (int j = 0; j < kGroupTiles; j++)
                            if (j < gt)
                                mma_f8f6f4(d0 + (uint32_t)(j * HI),
                                           adesc + (uint64_t)((j * kTileBytes) >> 4) + 2 * kk,
                                           bdesc + 2 * kk, kIdesc, kk > 0 ? 1u : 0u);
                    }
                    mma_commit(&empty[stage]);
                    mma_commit(&accfull[set]);
                    ng++;
                    if (++stage == kStages) {
                        stage = 0;
                        sphase ^= 1;
                    }
                }
            }
            // drain: all issued MMAs complete before TMEM is released
            mma_commit(drain);
            mbar_drain(drain, 0, a.st);
        }
    } else if (warp == 2) {
        // ---------------- item prefetch ----------------
        int nit = 0;
        for (int ii = 0; ii < n_my; ii++) {
            Item x;
            if (!fetch_item(a, items, v0, v1, ii, x, lane == 0)) continue;
            const int slot = nit % kAux;
            if (!mbar_wait_warp(&auxempty[slot], ((nit / kAux) & 1) ^ 1, abort_flag, a.st)) break;
            float* ws_s = aux + slot * kAuxFloats;
            float* ks_s = ws_s + HI;
#pragma unroll
            for (int h = lane; h < HI; h += 32)
                ws_s[h] = h < a.hreal ? __ldg(a.w + (int64_t)x.q * a.hreal + h) *
                                            __ldg(a.qs + (int64_t)x.q * a.hreal + h)
                                      : 0.f;
            // all of the item's key scales in flight at once (one memory latency per item)
            const int64_t e0 = (int64_t)x.tile0 * kTileRows;
            const int nrows = x.ntiles * kTileRows;
            float v[kChunkTiles * kTileRows / 32];
            if constexpr (!PAGED) {
#pragma unroll
                for (int k = 0; k < kChunkTiles * kTileRows / 32; k++) {
                    const int j = lane + 32 * k;
                    v[k] = (j < nrows && e0 + j < x.n_vis) ? __ldg(a.ks + x.row0 + e0 + j) : 0.f;
                }
            } else {
                // block table: the rows of the item's blocks first (one per 32 entries), then
                // every scale load in flight at once
                int64_t r[kChunkTiles * kTileRows / 32];
#pragma unroll
                for (int k = 0; k < kChunkTiles * kTileRows / 32; k++) {
                    const int j = lane + 32 * k;
                    r[k] = (j < nrows && e0 + j < x.n_vis) ? a.er.row(x.b, e0 + j) : -1;
                }
#pragma unroll
                for (int k = 0; k < kChunkTiles * kTileRows / 32; k++)
                    v[k] = (r[k] >= 0 && r[k] < a.ent_rows) ? __ldg(a.ks + r[k]) : 0.f;
            }
#pragma unroll
            for (int k = 0; k < kChunkTiles * kTileRows / 32; k++)
                if (lane + 32 * k < nrows) ks_s[lane + 32 * k] = v[k];
            mbar_arrive(&auxfull[slot]);
            nit++;
        }
    } else {
        // ---------------- epilogue (warps 3..10) ----------------
        const int grp = (warp - kFirstEpiWarp) / 4;   // takes the group's tiles j % 2 == grp
        const int quarter = warp & 3;                 // TMEM lanes this warp may access
        const int row_in_tile = quarter * 32 + lane;
        int ng = 0, nit = 0;
        bool ok = true;
        bool waited = false;   // for the previous grid, before this thread's first store
        for (int ii = 0; ii < n_my && ok; ii++) {
            Item x;
            if (!fetch_item(a, items, v0, v1, ii, x, false)) continue;
            const int slot = nit % kAux;
            if (!mbar_wait_warp(&auxfull[slot], (nit / kAux) & 1, abort_flag, a.st)) break;
            const float* ws_s = aux + slot * kAuxFloats;
            const float* ks_s = ws_s + HI;
            float ws[HI];
#pragma unroll
            for (int h = 0; h < HI; h += 4) {
                const float4 v4 = *reinterpret_cast<const float4*>(ws_s + h);
                ws[h] = v4.x;
                ws[h + 1] = v4.y;
                ws[h + 2] = v4.z;
                ws[h + 3] = v4.w;
            }
            float* srow = a.scores + (int64_t)x.q * a.ld;
            for (int g0 = 0; g0 < x.ntiles; g0 += kGroupTiles) {
                const int gt = min(kGroupTiles, x.ntiles - g0);
                const int set = ng & (kAccSets - 1);
                if (!mbar_wait_warp(&accfull[set], (ng / kAccSets) & 1, abort_flag, a.st)) {
                    ok = false;
                    break;
                }
                tc_fence_after();
                if (!waited) {
                    pdl_wait();
                    waited = true;
                }
                for (int j = grp; j < gt; j += 2) {
                    const int tt = g0 + j;
                    const int e = (x.tile0 + tt) * kTileRows + row_in_tile;
                    uint32_t d[HI];
                    const uint32_t taddr = tmem_base + ((uint32_t)(quarter * 32) << 16) +
                                           (uint32_t)((set * kGroupTiles + j) * HI);
                    if constexpr (HI == 64) {
                        tmem_ld64(taddr, d);
                    } else if constexpr (HI == 32) {
                        tmem_ld32(taddr, d);
                    } else {
                        tmem_ld16(taddr, d);
                    }
                    tmem_ld_wait();
                    uint32_t key = 0u;   // below every score's key
                    if (e < x.n_vis) {
                        float acc = 0.f;
#pragma unroll
                        for (int h = 0; h < HI; h++)
                            acc = fmaf(ws[h], fmaxf(__uint_as_float(d[h]), 0.f), acc);
                        const float sc = acc * ks_s[tt * kTileRows + row_in_tile];
                        if (sc != sc) flag(a.st, CSA_DEV_NAN);
                        srow[e] = sc;
                        key = order_key(sc);
                    }
                    if (a.gmax) {
                        // the warp's 32 rows are one group of 32 consecutive entries
                        key = __reduce_max_sync(0xffffffffu, key);
                        const int e0 = e - lane;
                        if (lane == 0 && e0 < x.n_vis) a.gmax[(int64_t)x.q * a.ld_g + (e0 >> 5)] = key;
                    }
                }
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(&accempty[set]);
                ng++;
            }
            __syncwarp();
            if (lane == 0) mbar_arrive(&auxempty[slot]);
            nit++;
        }
    }

    pdl_wait();
    tc_fence_before();
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem_base, tmem_cols<HI>());
    }
}

template <int HI, int DI>
size_t smem_bytes() {
    return 1024 + kStages * kGroupTiles * tile_bytes<DI>() + 2 * HI * DI + kAux * aux_floats<HI>() * sizeof(float) +
           (2 * kStages + 4 + 2 * kAccSets + 2 * kAux + 1) * 8 + 16 + kMaxItems * sizeof(Item);
}

using EncodeFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                              const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                              const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                              CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeFn get_encode_fn() {
    static EncodeFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void* p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeFn>(p);
    });
    return fn;
}

// Row-major [rows x dI] byte matrix (dI 64 or 128), boxes of box_rows x dI bytes, swizzled
// by the row width (128- or 64-byte swizzle).
bool make_rows_map(CUtensorMap* m, const void* base, uint64_t rows, uint32_t box_rows, int dI) {
    EncodeFn enc = get_encode_fn();
    if (!enc) return false;
    const cuuint64_t dims[2] = {(cuuint64_t)dI, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)dI};
    const cuuint32_t box[2] = {(cuuint32_t)dI, box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return enc(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
               estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
               dI == 128 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) ==
           CUDA_SUCCESS;
}

int num_sms() {
    static int n = 0;
    if (n == 0) {
        int dev = 0;
        cudaGetDevice(&dev);
        cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
        if (n <= 0) n = 148;
    }
    return n;
}

template <int HI, int DI>
cudaError_t launch_hi(const uint8_t* qI, const uint8_t* kI, const IdxArgs& args,
                      cudaStream_t stream) {
    CUtensorMap mk, mq;
    if (!make_rows_map(&mk, kI, (uint64_t)args.ent_rows, args.er.bt ? kPageRows : kTileRows, DI) ||
        !make_rows_map(&mq, qI, (uint64_t)args.Q * args.hreal, (uint32_t)args.hreal, DI))
        return cudaErrorInvalidValue;
    const size_t sm = smem_bytes<HI, DI>();
    auto kernel = args.er.bt ? indexer_tc_kernel<HI, DI, true> : indexer_tc_kernel<HI, DI, false>;
    cudaError_t e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)sm);
    if (e != cudaSuccess) return e;
    const int64_t tiles = (int64_t)args.Q * args.qtiles;
    const int grid = (int)(tiles < (int64_t)num_sms() ? tiles : (int64_t)num_sms());
    LaunchScope scope(kKIndexerTc, stream);
    return launch_pdl(kernel, dim3(grid), dim3(kThreads), sm, stream, mk, mq, args);
}

}  // namespace

// Any head count 1..64 (run on the MMA width 16, 32 or 64 at or above it), dim 64 or 128.
bool indexer_tc_supported(int HI, int dI) {
    return (dI == 64 || dI == 128) && HI >= 1 && HI <= 64;
}

cudaError_t launch_indexer_tc(const uint8_t* qI, const float* qs, const float* w,
                              const uint8_t* kI, const float* ks, int64_t ent_rows,
                              const int64_t* seq_len, const EntryRows& er,
                              const int32_t* q_seq, const int32_t* q_pos, int Q, int B, int HI,
                              int dI, int m, int max_n, float* scores, int64_t ld, int32_t* st,
                              cudaStream_t stream, uint32_t* gmax, int64_t ld_g) {
    if (Q == 0 || max_n == 0 || ent_rows == 0) return cudaSuccess;
    IdxArgs args;
    args.qs = qs;
    args.w = w;
    args.ks = ks;
    args.seq_len = seq_len;
    args.er = er;
    args.q_seq = q_seq;
    args.q_pos = q_pos;
    args.scores = scores;
    args.ld = ld;
    args.ent_rows = ent_rows;
    args.st = st;
    args.Q = Q;
    args.B = B;
    args.m = m;
    args.max_n = max_n;
    args.hreal = HI;
    args.keys_once = Q <= B;
    args.gmax = gmax;
    args.ld_g = ld_g;
    args.qtiles = (max_n + kTileRows - 1) / kTileRows;
    args.chunks_per_q = (args.qtiles + kChunkTiles - 1) / kChunkTiles;
    if (!indexer_tc_supported(HI, dI)) return cudaErrorInvalidValue;
    const int width = HI <= 16 ? 16 : HI <= 32 ? 32 : 64;   // MMA N
    if (dI == 128) {
        switch (width) {
            case 64: return launch_hi<64, 128>(qI, kI, args, stream);
            case 32: return launch_hi<32, 128>(qI, kI, args, stream);
            default: return launch_hi<16, 128>(qI, kI, args, stream);
        }
    }
    switch (width) {
        case 64: return launch_hi<64, 64>(qI, kI, args, stream);
        case 32: return launch_hi<32, 64>(qI, kI, args, stream);
        default: return launch_hi<16, 64>(qI, kI, args, stream);
    }
}

}  // namespace csa
